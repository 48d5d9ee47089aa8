// Materialised MTA forward: the T x T maps of one call live in the workspace.
//
// Four kernels, one per group of steps of "Multi-Token Attention -- Paper
// Graph", section 3.4, all arithmetic in fp32 on CUDA cores:
//   k_logits        S1 + S2   A0 = Mask_0(Q K^T / sqrt(d))      -> map0
//   k_conv          S3 (+S4)  C = Conv2d_theta(A0), Eq. (4)/(5) -> map1
//   k_softmax_mix   S5 + S6   softmax rows, post-softmax head mix (Eq. (7))
//                             -> map0 (A0 is dead by then)
//   k_pv_groupnorm  S7..S9    A_new V, per-head GroupNorm with warp-shuffle
//                             reductions, depth scale -> out
// Only entries with key j <= query i are written or read; the maps hold
// garbage above the diagonal.  This path is the measured stepping stone and
// the general fallback (fp32 I/O, shapes the fused kernel does not take).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "io.cuh"
#include "mta_internal.h"

namespace mta {
namespace {

constexpr int kLogitTile = 64;   // k_logits: 64 x 64 output tile
constexpr int kLogitDk = 32;     // contraction chunk
constexpr int kConvRows = 32;    // k_conv: 32 x 64 output tile
constexpr int kConvCols = 64;
constexpr int kMaxCq = 8;
constexpr int kMaxCk = 15;
constexpr int kPvRows = 32;      // k_pv_groupnorm: 32 query rows x d
constexpr int kPvKeys = 32;
constexpr int kMaxD = 128;

// S1 + S2: map0[bh][i][j] = (j <= i) ? q_i . k_j * scale : 0 on tiles that
// touch the causal triangle.  Grid (col tiles, row tiles, B*H), 256 threads,
// each thread a 4 x 4 block of the 64 x 64 tile.
template <typename TIO>
__global__ void __launch_bounds__(256)
k_logits(const TIO *__restrict__ q, const TIO *__restrict__ k, float *__restrict__ map0,
         int T, int d, float scale)
{
    const int ct = blockIdx.x, rt = blockIdx.y;
    if (ct > rt) return;                     // the whole tile lies above the diagonal
    const size_t bh = blockIdx.z;
    const int i0 = rt * kLogitTile, j0 = ct * kLogitTile;
    __shared__ float qs[kLogitDk][kLogitTile + 1];
    __shared__ float ks[kLogitDk][kLogitTile + 1];
    const int tid = threadIdx.x;
    const int tx = tid % 16, ty = tid / 16;
    float acc[4][4] = {};
    const TIO *qb = q + bh * (size_t)T * d;
    const TIO *kb = k + bh * (size_t)T * d;
    for (int e0 = 0; e0 < d; e0 += kLogitDk) {
        for (int idx = tid; idx < kLogitTile * kLogitDk; idx += 256) {
            int r = idx / kLogitDk, e = idx % kLogitDk;
            int gi = i0 + r, gj = j0 + r, ge = e0 + e;
            qs[e][r] = (gi < T && ge < d) ? to_f32(qb[(size_t)gi * d + ge]) : 0.f;
            ks[e][r] = (gj < T && ge < d) ? to_f32(kb[(size_t)gj * d + ge]) : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int e = 0; e < kLogitDk; ++e) {
            float a[4], b[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) { a[u] = qs[e][ty * 4 + u]; b[u] = ks[e][tx * 4 + u]; }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(a[u], b[w], acc[u][w]);
        }
        __syncthreads();
    }
    float *mb = map0 + bh * (size_t)T * T;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        int i = i0 + ty * 4 + u;
        if (i >= T) continue;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            int j = j0 + tx * 4 + w;
            if (j >= T) continue;
            mb[(size_t)i * T + j] = (j <= i) ? acc[u][w] * scale : 0.f;
        }
    }
}

// S3 (+S4): map1[bh][i][j] = sum_{i',j'} theta[i'][j'] A0[i-i'][j-j'] for
// j <= i.  The 32 x 64 output tile reads a (32 + c_q - 1) x (64 + c_k - 1)
// halo of A0 into shared memory; reads outside [0,T) or above the diagonal
// (c > r) are the zeros of Mask_0 and of the zero padding.
__global__ void __launch_bounds__(256)
k_conv(const float *__restrict__ map0, float *__restrict__ map1, const float *__restrict__ w_kq,
       int T, int H, int c_q, int c_k)
{
    const int i0 = blockIdx.y * kConvRows, j0 = blockIdx.x * kConvCols;
    if (j0 > i0 + kConvRows - 1) return;     // tile entirely above the diagonal
    const size_t bh = blockIdx.z;
    const int h = (int)(bh % H);
    __shared__ float tile[kConvRows + kMaxCq - 1][kConvCols + kMaxCk - 1 + 1];
    __shared__ float th[kMaxCq * kMaxCk];
    const int tid = threadIdx.x;
    const int L = (c_k + 1) / 2 - 1;         // keys reached to the left
    const int rows = kConvRows + c_q - 1, cols = kConvCols + c_k - 1;
    const float *mb = map0 + bh * (size_t)T * T;
    for (int idx = tid; idx < rows * cols; idx += 256) {
        int rr = idx / cols, cc = idx % cols;
        int r = i0 - (c_q - 1) + rr, c = j0 - L + cc;
        tile[rr][cc] = (r >= 0 && r < T && c >= 0 && c <= r) ? mb[(size_t)r * T + c] : 0.f;
    }
    for (int idx = tid; idx < c_q * c_k; idx += 256) th[idx] = w_kq[(size_t)h * c_q * c_k + idx];
    __syncthreads();
    const int col = tid % kConvCols;
    const int rbase = (tid / kConvCols) * (kConvRows / 4);
    float *cb = map1 + bh * (size_t)T * T;
    const int j = j0 + col;
    for (int ro = rbase; ro < rbase + kConvRows / 4; ++ro) {
        const int i = i0 + ro;
        if (i >= T || j >= T || j > i) continue;
        float acc = 0.f;
        for (int ip = 0; ip < c_q; ++ip) {
            const float *trow = &tile[ro + c_q - 1 - ip][col + c_k - 1];
            const float *trow_th = &th[ip * c_k];
            for (int jj = 0; jj < c_k; ++jj) acc = fmaf(trow_th[jj], trow[-jj], acc);
        }
        cb[(size_t)i * T + j] = acc;
    }
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Block-wide (256 threads) reduction through shared memory.
template <bool kMax>
__device__ float block_reduce(float x, float *red) {
    x = kMax ? warp_max(x) : warp_sum(x);
    const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
    __syncthreads();
    if (lane == 0) red[warp] = x;
    __syncthreads();
    float r = red[0];
    for (int w = 1; w < 8; ++w) r = kMax ? fmaxf(r, red[w]) : r + red[w];
    return r;
}

// S5 + S6 for one (batch, group, query row i): softmax of each head's conv
// row over j <= i, then A^h_new = sum_h' w_g[h][h'] P^h'.  mode 0 writes
// A_new for j <= i into dst (the forward); mode 1 writes P (pre-mix) and
// mode 2 writes A_new, both with zeros for i < j < T (the debug view).
template <int CH>
__global__ void __launch_bounds__(256)
k_softmax_mix(const float *__restrict__ map1, float *__restrict__ dst,
              const float *__restrict__ w_head, int T, int H, int mode)
{
    const int i = blockIdx.x;
    const int bg = blockIdx.y;
    const int G = H / CH;
    const int b = bg / G, g = bg % G;
    __shared__ float red[8];
    __shared__ float wsm[CH * CH];
    for (int idx = threadIdx.x; idx < CH * CH; idx += 256) wsm[idx] = w_head[(size_t)g * CH * CH + idx];
    float m[CH], inv_l[CH];
    const float *rowp[CH];
    float *dstp[CH];
#pragma unroll
    for (int hh = 0; hh < CH; ++hh) {
        size_t bh = (size_t)b * H + g * CH + hh;
        rowp[hh] = map1 + (bh * T + i) * (size_t)T;
        dstp[hh] = dst + (bh * T + i) * (size_t)T;
    }
#pragma unroll
    for (int hh = 0; hh < CH; ++hh) {
        float mx = -INFINITY;
        for (int j = threadIdx.x; j <= i; j += 256) mx = fmaxf(mx, rowp[hh][j]);
        m[hh] = block_reduce<true>(mx, red);
        float sm = 0.f;
        for (int j = threadIdx.x; j <= i; j += 256) sm += expf(rowp[hh][j] - m[hh]);
        inv_l[hh] = 1.f / block_reduce<false>(sm, red);
    }
    __syncthreads();
    for (int j = threadIdx.x; j < T; j += 256) {
        if (j > i) {
            if (mode == 0) break;
#pragma unroll
            for (int hh = 0; hh < CH; ++hh) dstp[hh][j] = 0.f;
            continue;
        }
        float p[CH];
#pragma unroll
        for (int hh = 0; hh < CH; ++hh) p[hh] = expf(rowp[hh][j] - m[hh]) * inv_l[hh];
        if (mode == 1) {
#pragma unroll
            for (int hh = 0; hh < CH; ++hh) dstp[hh][j] = p[hh];
            continue;
        }
#pragma unroll
        for (int ho = 0; ho < CH; ++ho) {
            float a = 0.f;
#pragma unroll
            for (int hi = 0; hi < CH; ++hi) a = fmaf(wsm[ho * CH + hi], p[hi], a);
            dstp[ho][j] = a;
        }
    }
}

// S7..S9: O = A_new V for 32 query rows of one (b, h) and all d columns,
// then per row: mean and biased variance over d (warp-shuffle reductions),
// out = scale_h * ((O - mean) / sqrt(var + eps) * gamma + beta), with scale_h
// the depth scale or, with a gate, sigmoid(g_h) ("Group Normalization with
// Sigmoid Gating").
template <typename TIO>
__global__ void __launch_bounds__(256)
k_pv_groupnorm(const float *__restrict__ amap, const TIO *__restrict__ v,
               const float *__restrict__ gn_weight, const float *__restrict__ gn_bias,
               float depth_scale, const float *__restrict__ gate, float eps,
               TIO *__restrict__ out, int T, int H, int d)
{
    const int i0 = blockIdx.x * kPvRows;
    const size_t bh = blockIdx.y;
    const int b = (int)(bh / H), h = (int)(bh % H);
    __shared__ float as[kPvRows][kPvKeys + 1];
    __shared__ float vs[kPvKeys][kMaxD];
    __shared__ float os[kPvRows][kMaxD + 1];
    const int tid = threadIdx.x;
    const int rg = tid / 32;                 // rows rg*4 .. rg*4+3
    const int cg = (tid % 32) * 4;           // columns cg .. cg+3
    float acc[4][4] = {};
    const float *ab = amap + bh * (size_t)T * T;
    const TIO *vb = v + bh * (size_t)T * d;
    const int jend = min(T, i0 + kPvRows);   // keys beyond the last row are masked
    for (int j0 = 0; j0 < jend; j0 += kPvKeys) {
        for (int idx = tid; idx < kPvRows * kPvKeys; idx += 256) {
            int r = idx / kPvKeys, c = idx % kPvKeys;
            int i = i0 + r, j = j0 + c;
            as[r][c] = (i < T && j <= i) ? ab[(size_t)i * T + j] : 0.f;
        }
        for (int idx = tid; idx < kPvKeys * d; idx += 256) {
            int r = idx / d, e = idx % d;
            int j = j0 + r;
            vs[r][e] = (j < T) ? to_f32(vb[(size_t)j * d + e]) : 0.f;
        }
        __syncthreads();
        if (cg < d) {
#pragma unroll 4
            for (int c = 0; c < kPvKeys; ++c) {
                float x[4], y[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) { x[u] = as[rg * 4 + u][c]; y[u] = vs[c][cg + u]; }
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(x[u], y[w], acc[u][w]);
            }
        }
        __syncthreads();
    }
    if (cg < d) {
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int w = 0; w < 4; ++w) os[rg * 4 + u][cg + w] = acc[u][w];
    }
    __syncthreads();
    // one warp per row: warp rg owns rows rg*4 .. rg*4+3
    const int lane = tid % 32;
    for (int u = 0; u < 4; ++u) {
        const int r = rg * 4 + u, i = i0 + r;
        if (i >= T) continue;
        float s = 0.f;
        for (int e = lane; e < d; e += 32) s += os[r][e];
        const float mean = warp_sum(s) / d;
        float s2 = 0.f;
        for (int e = lane; e < d; e += 32) { float t = os[r][e] - mean; s2 += t * t; }
        const float var = warp_sum(s2) / d;
        const float inv = 1.f / sqrtf(var + eps);
        const float scale = gate ? 1.f / (1.f + expf(-gate[h])) : depth_scale;
        TIO *dst = out + ((size_t)b * T + i) * ((size_t)H * d) + (size_t)h * d;
        for (int e = lane; e < d; e += 32) {
            const size_t ch = (size_t)h * d + e;
            dst[e] = from_f32<TIO>(scale * ((os[r][e] - mean) * inv * gn_weight[ch] + gn_bias[ch]));
        }
    }
}

template <int CH>
void launch_softmax_mix(const mta_shape &s, const float *map1, float *dst, const float *w_head,
                        int mode, cudaStream_t st)
{
    dim3 grid(s.T, s.B * (s.H / CH));
    k_softmax_mix<CH><<<grid, 256, 0, st>>>(map1, dst, w_head, s.T, s.H, mode);
}

mta_status softmax_mix(const mta_shape &s, const float *map1, float *dst, const float *w_head,
                       int mode, cudaStream_t st)
{
    switch (s.c_h) {
        case 1: launch_softmax_mix<1>(s, map1, dst, w_head, mode, st); break;
        case 2: launch_softmax_mix<2>(s, map1, dst, w_head, mode, st); break;
        case 4: launch_softmax_mix<4>(s, map1, dst, w_head, mode, st); break;
        case 8: launch_softmax_mix<8>(s, map1, dst, w_head, mode, st); break;
        case 16: launch_softmax_mix<16>(s, map1, dst, w_head, mode, st); break;
        default: return MTA_ERR_UNSUPPORTED;
    }
    return MTA_OK;
}

template <typename TIO>
void logits_and_conv(const mta_shape &s, const void *q, const void *k, const float *w_kq,
                     float *map0, float *map1, cudaStream_t st, const Trace &tr)
{
    const int nt = (s.T + kLogitTile - 1) / kLogitTile;
    dim3 g1(nt, nt, s.B * s.H);
    tr.before(0, st);
    k_logits<TIO><<<g1, 256, 0, st>>>((const TIO *)q, (const TIO *)k, map0, s.T, s.d,
                                      1.0f / sqrtf((float)s.d));
    tr.after(0, st);
    dim3 g2((s.T + kConvCols - 1) / kConvCols, (s.T + kConvRows - 1) / kConvRows, s.B * s.H);
    tr.before(1, st);
    k_conv<<<g2, 256, 0, st>>>(map0, map1, w_kq, s.T, s.H, s.c_q, s.c_k);
    tr.after(1, st);
}

}  // namespace

const char *const kUnfusedKernelNames[kUnfusedKernels] = {"k_logits", "k_conv",
                                                         "k_softmax_mix", "k_pv_groupnorm"};

size_t unfused_workspace_bytes(const mta_shape &s) { return 2 * bh_tt(s) * sizeof(float); }

mta_status launch_unfused(const mta_shape &s, const ForwardArgs &a, void *ws, cudaStream_t st,
                          const Trace &tr)
{
    float *map0 = (float *)ws;
    float *map1 = map0 + bh_tt(s);
    if (s.io == MTA_BF16)
        logits_and_conv<__nv_bfloat16>(s, a.q, a.k, a.w_kq, map0, map1, st, tr);
    else
        logits_and_conv<float>(s, a.q, a.k, a.w_kq, map0, map1, st, tr);
    tr.before(2, st);
    mta_status rc = softmax_mix(s, map1, map0, a.w_head, 0, st);
    tr.after(2, st);
    if (rc != MTA_OK) return rc;
    dim3 g4((s.T + kPvRows - 1) / kPvRows, s.B * s.H);
    tr.before(3, st);
    if (s.io == MTA_BF16)
        k_pv_groupnorm<__nv_bfloat16><<<g4, 256, 0, st>>>(
            map0, (const __nv_bfloat16 *)a.v, a.gn_weight, a.gn_bias, a.depth_scale, a.gate,
            s.gn_eps, (__nv_bfloat16 *)a.out, s.T, s.H, s.d);
    else
        k_pv_groupnorm<float><<<g4, 256, 0, st>>>(map0, (const float *)a.v, a.gn_weight,
                                                  a.gn_bias, a.depth_scale, a.gate, s.gn_eps,
                                                  (float *)a.out, s.T, s.H, s.d);
    tr.after(3, st);
    return cudaGetLastError() == cudaSuccess ? MTA_OK : MTA_ERR_CUDA;
}

mta_status launch_debug_attention(const mta_shape &s, const void *q, const void *k,
                                  const float *w_kq, const float *w_head, float *attn, int stage,
                                  void *ws, cudaStream_t st)
{
    float *map0 = (float *)ws;
    float *map1 = map0 + bh_tt(s);
    const Trace none;
    if (s.io == MTA_BF16)
        logits_and_conv<__nv_bfloat16>(s, q, k, w_kq, map0, map1, st, none);
    else
        logits_and_conv<float>(s, q, k, w_kq, map0, map1, st, none);
    mta_status rc = softmax_mix(s, map1, attn, w_head, stage == 0 ? 1 : 2, st);
    if (rc != MTA_OK) return rc;
    return cudaGetLastError() == cudaSuccess ? MTA_OK : MTA_ERR_CUDA;
}

}  // namespace mta
