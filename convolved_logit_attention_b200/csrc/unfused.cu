// Materialised MTA forward: the T x T maps of one call live in the workspace.
//
// One kernel per group of steps of "Multi-Token Attention -- Paper Graph",
// section 3.4, all arithmetic in fp32 on CUDA cores (for bf16 I/O at d = 64
// or 128, k_logits and k_pv_groupnorm give way to the tcgen05 kernels of
// unfused_tc.cu):
//   k_logits        S1 + S2   A0 = Mask_0(Q K^T / sqrt(d))      -> map0
//   k_conv          S3 (+S4)  C = Conv2d_theta(A0), Eq. (4)/(5) -> map1
//   k_softmax_mix   S5 + S6   softmax rows, post-softmax head mix (Eq. (7))
//                             -> map0 (A0 is dead by then)
//   k_pv_groupnorm  S7..S9    A_new V, per-head GroupNorm with warp-shuffle
//                             reductions, depth scale -> out
// The compositions of "Putting Everything Together: The Full MTA Module"
// reuse the chain: k_conv with a second kernel on the probabilities (the
// post-softmax variant of "Key-Query Convolution", its Mask_0 being the
// j <= i rule below) and k_head_mix, a second head mix without a softmax.
// Steps a composition leaves out are skipped; the maps alternate.
// Only entries with key j <= query i are written or read; the maps hold
// garbage above the diagonal.  This path is the measured stepping stone and
// the general fallback (fp32 I/O, shapes the fused kernel does not take).
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>

#include "io.cuh"
#include "tc_util.cuh"
#include "mta_internal.h"

namespace mta {
namespace {

constexpr int kLogitTile = 128;  // k_logits: 128 x 128 output tile
constexpr int kLogitDk = 16;     // contraction chunk
constexpr int kLogitStride = kLogitTile + 4;
constexpr int kConvRows = 32;    // k_conv: 32 x 128 output tile
constexpr int kConvCols = 128;
constexpr int kConvStride = 164; // k_conv halo row stride (floats), 4 (mod 32)
constexpr int kMaxCq = 8;
constexpr int kMaxCk = 15;
constexpr int kPvRows = 64;      // k_pv_groupnorm: 64 query rows x d
constexpr int kPvKeys = 32;
constexpr int kPvAStride = kPvRows + 4;   // transposed attention chunk: key-major rows
constexpr int kMaxD = 128;

// S1 + S2: map0[bh][i][j] = (j <= i + band) ? q_i . k_j * scale : 0 on tiles
// that touch the causal triangle widened by `band` keys: band = 0 is Mask_0;
// the exact indicator of Eq. (4) needs the c_q - 1 keys past each query
// (band = c_q - 1), which the convolution's taps of later queries may read.  Grid (col tiles, row tiles, B*H), 256 threads,
// 128 x 128 tiles.  Thread (tx, ty) = (tid % 16, tid / 16) owns rows
// {ty*4 .. ty*4+3} and {64+ty*4 .. 64+ty*4+3} and the same pattern of
// columns with tx, so that its operands for one contraction index are four
// 16-byte shared loads (eight lanes of a warp read 128 contiguous bytes) for
// 64 FMAs.  Chunks of 16 contraction indices are staged transposed.
template <typename TQ, typename TK>
__global__ void __launch_bounds__(256)
k_logits(const TQ *__restrict__ q, const TK *__restrict__ k, float *__restrict__ map0,
         int T, int d, float scale, int band)
{
    const int ct = blockIdx.x, rt = blockIdx.y;
    const int i0 = rt * kLogitTile, j0 = ct * kLogitTile;
    if (j0 > i0 + kLogitTile - 1 + band) return;   // the whole tile lies past the band
    const size_t bh = blockIdx.z;
    __shared__ __align__(16) float qs[kLogitDk * kLogitStride];
    __shared__ __align__(16) float ks[kLogitDk * kLogitStride];
    const int tid = threadIdx.x;
    const int tx = tid % 16, ty = tid / 16;
    float acc[8][8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int w = 0; w < 8; ++w) acc[u][w] = 0.f;
    const TQ *qb = q + bh * (size_t)T * d;
    const TK *kb = k + bh * (size_t)T * d;
    for (int e0 = 0; e0 < d; e0 += kLogitDk) {
        for (int idx = tid; idx < kLogitTile * kLogitDk; idx += 256) {
            const int r = idx / kLogitDk, e = idx % kLogitDk;
            const int gi = i0 + r, gj = j0 + r, ge = e0 + e;
            qs[e * kLogitStride + r] = (gi < T && ge < d) ? to_f32(qb[(size_t)gi * d + ge]) : 0.f;
            ks[e * kLogitStride + r] = (gj < T && ge < d) ? to_f32(kb[(size_t)gj * d + ge]) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int e = 0; e < kLogitDk; ++e) {
            const float *qe = qs + e * kLogitStride, *ke = ks + e * kLogitStride;
            const float4 a0 = *reinterpret_cast<const float4 *>(qe + ty * 4);
            const float4 a1 = *reinterpret_cast<const float4 *>(qe + 64 + ty * 4);
            const float4 b0 = *reinterpret_cast<const float4 *>(ke + tx * 4);
            const float4 b1 = *reinterpret_cast<const float4 *>(ke + 64 + tx * 4);
            const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int u = 0; u < 8; ++u)
#pragma unroll
                for (int w = 0; w < 8; ++w) acc[u][w] = fmaf(a[u], bb[w], acc[u][w]);
        }
        __syncthreads();
    }
    float *mb = map0 + bh * (size_t)T * T;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const int i = i0 + (u < 4 ? ty * 4 + u : 64 + ty * 4 + u - 4);
        if (i >= T) continue;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int jb = j0 + half * 64 + tx * 4;
            float x[4];
#pragma unroll
            for (int w = 0; w < 4; ++w)
                x[w] = (jb + w <= i + band) ? acc[u][half * 4 + w] * scale : 0.f;
            if ((T & 3) == 0) {
                if (jb < T)
                    *reinterpret_cast<float4 *>(mb + (size_t)i * T + jb) =
                        make_float4(x[0], x[1], x[2], x[3]);
            } else {
#pragma unroll
                for (int w = 0; w < 4; ++w)
                    if (jb + w < T) mb[(size_t)i * T + jb + w] = x[w];
            }
        }
    }
}

// S3 (+S4): dst[bh][i][j] = sum_{i',j'} theta[i'][j'] src[i-i'][j-j'] for
// j <= i (also the post-softmax conv of the probabilities).  The 32 x 128
// output tile reads a (32 + c_q - 1)-row halo of src into shared memory
// (with T a multiple of 4, as cp.async copies of the 16-byte groups that
// hold it, so the halo starts at the group of key j0 - L and a thread's
// segment starts kOff columns later); reads outside [0,T) or above the
// diagonal (c > r) are the zeros of Mask_0 and of the zero padding: groups
// outside are zero-filled by the copy, and in a tile whose halo reaches the
// diagonal the keys past it are cleared after the copies land.  With kExact (the exact indicator of Eq. (4))
// the halo keeps src[r][c] for c <= r + band, and each output row i zeroes
// the keys c > i of the segments it reads: a tap (i', j') then adds
// src[i-i'][j-j'] exactly when j - j' <= i.  With nin > 1 (the 3-D
// convolution of "Putting Everything Together", nin = c_h) output head h
// sums the convs of the nin heads of its group, with the kernel
// w[(h * nin + hi)][c_q][c_k] for input head hi, one halo after another.  Thread (warp w, lane l) owns output row l and
// the 16 columns 16w .. 16w+15: per query tap i' it loads the row segment
// those columns reach (16 + c_k - 1 values) and the tap row theta[i'][*]
// with 16-byte shared loads into registers and applies the c_k key taps from
// there (c_k is a template parameter), so that shared loads stay far below
// the FMA count.  Halo rows are kConvStride floats apart, 4 (mod 32) banks,
// so the 16-byte loads of 8 consecutive rows hit distinct banks.  The taps
// accumulate in the order i' then j' for every output.
template <int CK, bool kExact, bool kMulti>
__global__ void __launch_bounds__(256, kExact || kMulti ? 4 : 5)
k_conv(const float *__restrict__ src, float *__restrict__ dst, const float *__restrict__ w_kq,
       int T, int H, int c_q, int band, int nin_arg)
{
    const int nin = kMulti ? nin_arg : 1;         // a compile-time 1 for the 2-D kernels
    constexpr int NC = kConvCols / 8;             // output columns per thread
    constexpr int CKP = (CK + 3) / 4 * 4;         // padded tap row
    constexpr int L = (CK + 1) / 2 - 1;           // keys reached to the left
    // With 16-byte copies the halo starts at the aligned group that holds key
    // j0 - L: halo column x is key j0 - L - kOff + x
    constexpr int kOff = ((-L) % 4 + 4) % 4;
    constexpr int NV = (kOff + CK + NC - 1 + 3) / 4;   // float4 loads per row segment
    constexpr int kLoadCols = 7 * NC + 4 * NV;    // halo columns any thread reads
    static_assert(kLoadCols <= kConvStride && kLoadCols >= kOff + kConvCols + CK - 1, "halo width");
    constexpr int NQ = kLoadCols / 4;             // 16-byte groups per halo row
    const int i0 = blockIdx.y * kConvRows, j0 = blockIdx.x * kConvCols;
    if (j0 > i0 + kConvRows - 1) return;          // tile entirely above the diagonal
    const size_t bh = blockIdx.z;
    const int h = (int)(bh % H);
    const size_t b = kMulti ? bh / H : 0;
    __shared__ __align__(16) float tile[(kConvRows + kMaxCq - 1) * kConvStride];
    static_assert(kMaxCk <= 16, "tap rows are padded to 16 floats");
    __shared__ __align__(16) float th[kMaxCq * 16];
    const int tid = threadIdx.x;
    const int rows = kConvRows + c_q - 1;
    const int ro = tid % 32;                      // output row within the tile
    const int c0 = (tid / 32) * NC;               // first of the thread's output columns
    float acc[NC];
#pragma unroll
    for (int u = 0; u < NC; ++u) acc[u] = 0.f;
    for (int hi = 0; hi < nin; ++hi) {
        // input head and kernel block (h's own for the 2-D kernels)
        const float *mb = src + (kMulti ? b * H + (h / nin) * nin + hi : bh) * (size_t)T * T;
        const float *wk = w_kq + (kMulti ? (size_t)h * nin + hi : (size_t)h) * c_q * CK;
        if (hi > 0) __syncthreads();              // every thread is done with the last halo
        const int cbase = j0 - L - kOff;          // key of halo column 0
        if ((T & 3) == 0) {
            // cp.async copies of the 16-byte groups of the halo; a group is
            // either inside [0, T) or outside it, and one outside (or starting
            // past the band) is zero-filled
            for (int idx = tid; idx < rows * NQ; idx += 256) {
                const int rr = idx / NQ, qq = idx % NQ;
                const int r = i0 - (c_q - 1) + rr, c = cbase + 4 * qq;
                const bool in = r >= 0 && r < T && c >= 0 && c < T && c <= r + band;
                tc::cp_async16(&tile[rr * kConvStride + 4 * qq], mb + (in ? (size_t)r * T + c : 0), in);
            }
            tc::cp_async_wait_all();
            // keys past r + band inside a copied group must read zero (the map
            // is not written there): only tiles whose halo reaches the band
            if (cbase + kLoadCols - 1 > i0 - (c_q - 1) + band) {
                __syncthreads();
                for (int idx = tid; idx < rows * kLoadCols; idx += 256) {
                    const int rr = idx / kLoadCols, x = idx % kLoadCols;
                    if (cbase + x > i0 - (c_q - 1) + rr + band) tile[rr * kConvStride + x] = 0.f;
                }
            }
        } else {
            for (int idx = tid; idx < rows * kLoadCols; idx += 256) {
                const int rr = idx / kLoadCols, x = idx % kLoadCols;
                const int r = i0 - (c_q - 1) + rr, c = cbase + x;
                tile[rr * kConvStride + x] =
                    (r >= 0 && r < T && c >= 0 && c < T && c <= r + band) ? mb[(size_t)r * T + c]
                                                                          : 0.f;
            }
        }
        for (int idx = tid; idx < c_q * CKP; idx += 256) {
            const int ip = idx / CKP, jj = idx % CKP;
            th[idx] = jj < CK ? wk[(size_t)ip * CK + jj] : 0.f;
        }
        __syncthreads();
        for (int ip = 0; ip < c_q; ++ip) {
            const float4 *seg4 =
                reinterpret_cast<const float4 *>(&tile[(ro + c_q - 1 - ip) * kConvStride + c0]);
            float seg[4 * NV];
#pragma unroll
            for (int v = 0; v < NV; ++v) {
                const float4 t = seg4[v];
                seg[4 * v] = t.x; seg[4 * v + 1] = t.y; seg[4 * v + 2] = t.z; seg[4 * v + 3] = t.w;
            }
            if (kExact) {                         // the indicator: keys past query i read 0
                const int kfirst = cbase + c0;    // key of seg[0]
#pragma unroll
                for (int v = 0; v < 4 * NV; ++v)
                    if (kfirst + v > i0 + ro) seg[v] = 0.f;
            }
            const float4 *tr4 = reinterpret_cast<const float4 *>(&th[ip * CKP]);
            float tr[CKP];
#pragma unroll
            for (int v = 0; v < CKP / 4; ++v) {
                const float4 t = tr4[v];
                tr[4 * v] = t.x; tr[4 * v + 1] = t.y; tr[4 * v + 2] = t.z; tr[4 * v + 3] = t.w;
            }
#pragma unroll
            for (int jj = 0; jj < CK; ++jj)
#pragma unroll
                for (int u = 0; u < NC; ++u) acc[u] = fmaf(tr[jj], seg[kOff + CK - 1 - jj + u], acc[u]);
        }
    }
    const int i = i0 + ro;
    if (i >= T) return;
    float *row = dst + bh * (size_t)T * T + (size_t)i * T;
#pragma unroll
    for (int g = 0; g < NC / 4; ++g) {
        const int jb = j0 + c0 + 4 * g;
        if ((T & 3) == 0 && jb + 3 <= i && jb < T) {
            *reinterpret_cast<float4 *>(row + jb) =
                make_float4(acc[4 * g], acc[4 * g + 1], acc[4 * g + 2], acc[4 * g + 3]);
        } else {
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (jb + u < T && jb + u <= i) row[jb + u] = acc[4 * g + u];
        }
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
// row over j <= i, then A^h_new = sum_h' w_g[h][h'] P^h' (w_head null: the
// identity, no mixing).  mode 0 writes
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
    for (int idx = threadIdx.x; idx < CH * CH; idx += 256)
        wsm[idx] = w_head ? w_head[(size_t)g * CH * CH + idx] : (idx / CH == idx % CH ? 1.f : 0.f);
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

// Eq. (7) without a softmax, for one (batch, group, query row i):
// dst^h[i][j] = sum_h' w_g[h][h'] src^h'[i][j] for j <= i.  The second head
// mix of a repeated MTA convolution, applied to probabilities that the
// post-softmax key-query conv has already filtered.
constexpr float kLog2eF = 1.4426950408889634f;

__device__ __forceinline__ float exp2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// The forward's S5 + S6 (mode 0) with the row held in registers, for
// T <= 1024 * Q4 and T % 4 == 0: each thread loads its 16-byte groups of each
// of the c_h heads' rows once (keys past i read as -inf), the c_h row maxima
// and then the c_h sums of exponentials are reduced over the CTA together,
// and A_new is written from the registers.  One read of the row instead of
// three, two CTA reductions instead of 2 c_h.
template <int CH, int Q4>
__global__ void __launch_bounds__(256)
k_softmax_mix_reg(const float *__restrict__ map1, float *__restrict__ dst,
                  const float *__restrict__ w_head, int T, int H)
{
    const int i = blockIdx.x;
    const int bg = blockIdx.y;
    const int G = H / CH;
    const int b = bg / G, g = bg % G;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    __shared__ float red[8][CH];
    __shared__ float wsm[CH * CH];
    for (int idx = tid; idx < CH * CH; idx += 256)
        wsm[idx] = w_head ? w_head[(size_t)g * CH * CH + idx] : (idx / CH == idx % CH ? 1.f : 0.f);
    const int nq = (i + 4) / 4;                   // 16-byte groups holding keys 0 .. i
    float v[CH][Q4][4];
#pragma unroll
    for (int hh = 0; hh < CH; ++hh) {
        const size_t bh = (size_t)b * H + g * CH + hh;
        const float *rowp = map1 + (bh * T + i) * (size_t)T;
#pragma unroll
        for (int q = 0; q < Q4; ++q) {
            const int jq = tid + 256 * q;
            float4 t = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            if (jq < nq) t = *reinterpret_cast<const float4 *>(rowp + 4 * jq);
            v[hh][q][0] = 4 * jq <= i ? t.x : -INFINITY;
            v[hh][q][1] = 4 * jq + 1 <= i ? t.y : -INFINITY;
            v[hh][q][2] = 4 * jq + 2 <= i ? t.z : -INFINITY;
            v[hh][q][3] = 4 * jq + 3 <= i ? t.w : -INFINITY;
        }
    }
    float m[CH], inv_l[CH];
#pragma unroll
    for (int hh = 0; hh < CH; ++hh) {
        float mx = -INFINITY;
#pragma unroll
        for (int q = 0; q < Q4; ++q)
#pragma unroll
            for (int e = 0; e < 4; ++e) mx = fmaxf(mx, v[hh][q][e]);
        mx = warp_max(mx);
        if (lane == 0) red[warp][hh] = mx;
    }
    __syncthreads();
#pragma unroll
    for (int hh = 0; hh < CH; ++hh) {
        float r = red[0][hh];
        for (int w = 1; w < 8; ++w) r = fmaxf(r, red[w][hh]);
        m[hh] = r;
    }
    __syncthreads();                              // red is read by every thread before reuse
    // exp(x - m) as 2^((x - m) log2 e) with the hardware exp2 (ex2.approx, a
    // couple of ulp): the kernel is issue-bound with a full-precision expf
#pragma unroll
    for (int hh = 0; hh < CH; ++hh) {
        float sm = 0.f;
#pragma unroll
        for (int q = 0; q < Q4; ++q)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                v[hh][q][e] = exp2_approx((v[hh][q][e] - m[hh]) * kLog2eF);
                sm += v[hh][q][e];
            }
        sm = warp_sum(sm);
        if (lane == 0) red[warp][hh] = sm;
    }
    __syncthreads();
#pragma unroll
    for (int hh = 0; hh < CH; ++hh) {
        float r = red[0][hh];
        for (int w = 1; w < 8; ++w) r += red[w][hh];
        inv_l[hh] = 1.f / r;
    }
#pragma unroll
    for (int q = 0; q < Q4; ++q) {
        const int jq = tid + 256 * q;
        if (jq >= nq) break;
#pragma unroll
        for (int ho = 0; ho < CH; ++ho) {
            float a[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float acc = 0.f;
#pragma unroll
                for (int hi = 0; hi < CH; ++hi)
                    acc = fmaf(wsm[ho * CH + hi], v[hi][q][e] * inv_l[hi], acc);
                a[e] = acc;
            }
            const size_t bh = (size_t)b * H + g * CH + ho;
            *reinterpret_cast<float4 *>(dst + (bh * T + i) * (size_t)T + 4 * jq) =
                make_float4(a[0], a[1], a[2], a[3]);
        }
    }
}

template <int CH>
__global__ void __launch_bounds__(256)
k_head_mix(const float *__restrict__ src, float *__restrict__ dst,
           const float *__restrict__ w_head, int T, int H)
{
    const int i = blockIdx.x;
    const int bg = blockIdx.y;
    const int G = H / CH;
    const int b = bg / G, g = bg % G;
    __shared__ float wsm[CH * CH];
    for (int idx = threadIdx.x; idx < CH * CH; idx += 256) wsm[idx] = w_head[(size_t)g * CH * CH + idx];
    __syncthreads();
    const size_t bh0 = (size_t)b * H + (size_t)g * CH;
    for (int j = threadIdx.x; j <= i; j += 256) {
        float x[CH];
#pragma unroll
        for (int hh = 0; hh < CH; ++hh) x[hh] = src[((bh0 + hh) * T + i) * (size_t)T + j];
#pragma unroll
        for (int ho = 0; ho < CH; ++ho) {
            float a = 0.f;
#pragma unroll
            for (int hi = 0; hi < CH; ++hi) a = fmaf(wsm[ho * CH + hi], x[hi], a);
            dst[((bh0 + ho) * T + i) * (size_t)T + j] = a;
        }
    }
}

// S7..S9: O = A_new V for 64 query rows of one (b, h) and all d columns,
// then per row: mean and biased variance over d (warp-shuffle reductions),
// out = scale_h * ((O - mean) / sqrt(var + eps) * gamma + beta), with scale_h
// the depth scale or, with a gate, sigmoid(g_h) ("Group Normalization with
// Sigmoid Gating").  Thread (warp w, lane l) accumulates rows 8w .. 8w+7 and
// columns 4l .. 4l+3.  Each 32-key chunk of the attention rows is stored
// transposed (key-major), so that the 8 values a thread needs for one key
// are two 16-byte broadcast loads and its V values one 16-byte load: three
// shared loads per 32 FMAs.  Keys accumulate in increasing order.
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
    // the key loop's chunks, then (aliased) the finished O rows
    __shared__ __align__(16) float smem[kPvRows * (kMaxD + 1)];
    static_assert(kPvKeys * (kPvAStride + kMaxD) <= kPvRows * (kMaxD + 1), "smem carve");
    float *asT = smem;                             // [kPvKeys][kPvAStride]
    float *vs = smem + kPvKeys * kPvAStride;       // [kPvKeys][kMaxD]
    float *os = smem;                              // [kPvRows][kMaxD + 1]
    const int tid = threadIdx.x;
    const int rg = tid / 32;                       // rows rg*8 .. rg*8+7
    const int cg = (tid % 32) * 4;                 // columns cg .. cg+3
    float acc[8][4];
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[u][w] = 0.f;
    const float *ab = amap + bh * (size_t)T * T;
    const TIO *vb = v + bh * (size_t)T * d;
    const bool vec4 = (T & 3) == 0;               // attention rows 16-byte aligned
    const int jend = min(T, i0 + kPvRows);        // keys beyond the last row are masked
    for (int j0 = 0; j0 < jend; j0 += kPvKeys) {
        // attention chunk: thread (row r, keys 4q .. 4q+3), transposed into asT
        for (int idx = tid; idx < kPvRows * (kPvKeys / 4); idx += 256) {
            const int r = idx / (kPvKeys / 4), c = (idx % (kPvKeys / 4)) * 4;
            const int i = i0 + r, j = j0 + c;
            float x[4] = {0.f, 0.f, 0.f, 0.f};
            if (i < T) {
                const float *src = ab + (size_t)i * T + j;
                if (vec4 && j + 3 <= i) {
                    const float4 t = *reinterpret_cast<const float4 *>(src);
                    x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
                } else {
#pragma unroll
                    for (int u = 0; u < 4; ++u) x[u] = (j + u <= i) ? src[u] : 0.f;
                }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) asT[(c + u) * kPvAStride + r] = x[u];
        }
        // V chunk: thread (key r, columns 4q .. 4q+3); d is a multiple of 8
        for (int r = tid / 32; r < kPvKeys; r += 8) {
            const int j = j0 + r;
            for (int e = (tid % 32) * 4; e < d; e += 128) {
                float y[4] = {0.f, 0.f, 0.f, 0.f};
                if (j < T) load4_f32(vb + (size_t)j * d + e, y);
#pragma unroll
                for (int u = 0; u < 4; ++u) vs[r * kMaxD + e + u] = y[u];
            }
        }
        __syncthreads();
        if (cg < d) {
#pragma unroll 4
            for (int c = 0; c < kPvKeys; ++c) {
                const float4 xa = *reinterpret_cast<const float4 *>(&asT[c * kPvAStride + rg * 8]);
                const float4 xb =
                    *reinterpret_cast<const float4 *>(&asT[c * kPvAStride + rg * 8 + 4]);
                const float4 y = *reinterpret_cast<const float4 *>(&vs[c * kMaxD + cg]);
                const float x[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
                const float yy[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
                for (int u = 0; u < 8; ++u)
#pragma unroll
                    for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(x[u], yy[w], acc[u][w]);
            }
        }
        __syncthreads();
    }
    // every thread has passed the loop's last barrier: os may reuse the chunks
    if (cg < d) {
#pragma unroll
        for (int u = 0; u < 8; ++u)
#pragma unroll
            for (int w = 0; w < 4; ++w) os[(rg * 8 + u) * (kMaxD + 1) + cg + w] = acc[u][w];
    }
    __syncthreads();
    // one warp per row: warp rg owns rows rg*8 .. rg*8+7
    const int lane = tid % 32;
    const float scale = gate ? 1.f / (1.f + expf(-gate[h])) : depth_scale;
    for (int u = 0; u < 8; ++u) {
        const int r = rg * 8 + u, i = i0 + r;
        if (i >= T) continue;
        const float *orow = os + r * (kMaxD + 1);
        float s = 0.f;
        for (int e = lane; e < d; e += 32) s += orow[e];
        const float mean = warp_sum(s) / d;
        float s2 = 0.f;
        for (int e = lane; e < d; e += 32) { float t = orow[e] - mean; s2 += t * t; }
        const float var = warp_sum(s2) / d;
        const float inv = 1.f / sqrtf(var + eps);
        TIO *dst = out + ((size_t)b * T + i) * ((size_t)H * d) + (size_t)h * d;
        for (int e = lane; e < d; e += 32) {
            const size_t ch = (size_t)h * d + e;
            dst[e] = from_f32<TIO>(scale * ((orow[e] - mean) * inv * gn_weight[ch] + gn_bias[ch]));
        }
    }
}

}  // namespace

// Launchers of the chain's kernels, shared with the backward pass
// (backward.cu) through mta_internal.h.
template <int CH>
void launch_softmax_mix(const mta_shape &s, const float *map1, float *dst, const float *w_head,
                        int mode, cudaStream_t st)
{
    dim3 grid(s.T, s.B * (s.H / CH));
    if constexpr (CH <= 4) {
        if (mode == 0 && s.T % 4 == 0 && s.T <= 4096) {
            if (s.T <= 1024)
                k_softmax_mix_reg<CH, 1><<<grid, 256, 0, st>>>(map1, dst, w_head, s.T, s.H);
            else if (s.T <= 2048)
                k_softmax_mix_reg<CH, 2><<<grid, 256, 0, st>>>(map1, dst, w_head, s.T, s.H);
            else
                k_softmax_mix_reg<CH, 4><<<grid, 256, 0, st>>>(map1, dst, w_head, s.T, s.H);
            return;
        }
    }
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

template <int CH>
void launch_head_mix(const mta_shape &s, const float *src, float *dst, const float *w_head,
                     cudaStream_t st)
{
    dim3 grid(s.T, s.B * (s.H / CH));
    k_head_mix<CH><<<grid, 256, 0, st>>>(src, dst, w_head, s.T, s.H);
}

mta_status head_mix(const mta_shape &s, const float *src, float *dst, const float *w_head,
                    cudaStream_t st)
{
    switch (s.c_h) {
        case 1: launch_head_mix<1>(s, src, dst, w_head, st); break;
        case 2: launch_head_mix<2>(s, src, dst, w_head, st); break;
        case 4: launch_head_mix<4>(s, src, dst, w_head, st); break;
        case 8: launch_head_mix<8>(s, src, dst, w_head, st); break;
        case 16: launch_head_mix<16>(s, src, dst, w_head, st); break;
        default: return MTA_ERR_UNSUPPORTED;
    }
    return MTA_OK;
}

template <typename TQ, typename TK>
void launch_logits(const mta_shape &s, const void *q, const void *k, float *map0, float scale,
                   int band, cudaStream_t st)
{
    const int nt = (s.T + kLogitTile - 1) / kLogitTile;
    dim3 g1(nt, nt, s.B * s.H);
    k_logits<TQ, TK><<<g1, 256, 0, st>>>((const TQ *)q, (const TK *)k, map0, s.T, s.d, scale,
                                         band);
}

void launch_conv(const mta_shape &s, const float *src, float *dst, const float *w_kq, int band,
                 int nin, cudaStream_t st)
{
    dim3 g2((s.T + kConvCols - 1) / kConvCols, (s.T + kConvRows - 1) / kConvRows, s.B * s.H);
    switch (s.c_k) {
#define MTA_CONV_CASE(n) \
        case n:                                                                          \
            if (band > 0 && nin > 1)                                                     \
                k_conv<n, true, true><<<g2, 256, 0, st>>>(src, dst, w_kq, s.T, s.H, s.c_q,   \
                                                          band, nin);                    \
            else if (band > 0)                                                           \
                k_conv<n, true, false><<<g2, 256, 0, st>>>(src, dst, w_kq, s.T, s.H, s.c_q,  \
                                                           band, 1);                     \
            else if (nin > 1)                                                            \
                k_conv<n, false, true><<<g2, 256, 0, st>>>(src, dst, w_kq, s.T, s.H, s.c_q,  \
                                                           0, nin);                      \
            else                                                                         \
                k_conv<n, false, false><<<g2, 256, 0, st>>>(src, dst, w_kq, s.T, s.H, s.c_q, \
                                                            0, 1);                       \
            break;
        MTA_CONV_CASE(1) MTA_CONV_CASE(2) MTA_CONV_CASE(3) MTA_CONV_CASE(4) MTA_CONV_CASE(5)
        MTA_CONV_CASE(6) MTA_CONV_CASE(7) MTA_CONV_CASE(8) MTA_CONV_CASE(9) MTA_CONV_CASE(10)
        MTA_CONV_CASE(11) MTA_CONV_CASE(12) MTA_CONV_CASE(13) MTA_CONV_CASE(14) MTA_CONV_CASE(15)
#undef MTA_CONV_CASE
        default: break;   // c_k <= 15 is checked before any launch
    }
}

mta_status logits(const mta_shape &s, const void *q, const void *k, float *map0, int band,
                  cudaStream_t st)
{
    if (chain_tc_supported(s)) return logits_tc(s, q, k, map0, band, st);
    const float scale = 1.0f / sqrtf((float)s.d);
    if (s.io == MTA_BF16)
        launch_logits<__nv_bfloat16, __nv_bfloat16>(s, q, k, map0, scale, band, st);
    else
        launch_logits<float, float>(s, q, k, map0, scale, band, st);
    return MTA_OK;
}

void logits_f32_io(const mta_shape &s, const float *a, const void *b, float scale, float *map,
                   cudaStream_t st)
{
    if (s.io == MTA_BF16)
        launch_logits<float, __nv_bfloat16>(s, a, b, map, scale, 0, st);
    else
        launch_logits<float, float>(s, a, b, map, scale, 0, st);
}

namespace {

mta_status pv_groupnorm(const mta_shape &s, const float *amap, const ForwardArgs &a,
                        cudaStream_t st)
{
    if (chain_tc_supported(s)) return pv_groupnorm_tc(s, amap, a, st);
    dim3 g4((s.T + kPvRows - 1) / kPvRows, s.B * s.H);
    if (s.io == MTA_BF16)
        k_pv_groupnorm<__nv_bfloat16><<<g4, 256, 0, st>>>(
            amap, (const __nv_bfloat16 *)a.v, a.gn_weight, a.gn_bias, a.depth_scale, a.gate,
            s.gn_eps, (__nv_bfloat16 *)a.out, s.T, s.H, s.d);
    else
        k_pv_groupnorm<float><<<g4, 256, 0, st>>>(amap, (const float *)a.v, a.gn_weight,
                                                  a.gn_bias, a.depth_scale, a.gate, s.gn_eps,
                                                  (float *)a.out, s.T, s.H, s.d);
    return MTA_OK;
}

}  // namespace

const char *unfused_kernel_name(const mta_shape &s, int index)
{
    static const char *const fp32[kUnfusedKernels] = {"k_logits", "k_conv", "k_softmax_mix",
                                                      "k_pv_groupnorm"};
    static const char *const tc[kUnfusedKernels] = {"k_logits_tc", "k_conv", "k_softmax_mix",
                                                    "k_pv_groupnorm_tc"};
    if (index < 0 || index >= kUnfusedKernels) return nullptr;
    return chain_tc_supported(s) ? tc[index] : fp32[index];
}

size_t unfused_workspace_bytes(const mta_shape &s) { return 2 * bh_tt(s) * sizeof(float); }

int unfused_chain(const mta_shape &s, const ForwardArgs &a, const char **names)
{
    int n = 0;
    names[n++] = unfused_kernel_name(s, 0);
    if (a.w_kq || a.w_kq_3d) names[n++] = "k_conv";
    if (a.w_head_pre) names[n++] = "k_head_mix";
    names[n++] = "k_softmax_mix";
    if (a.w_kq_post) names[n++] = "k_conv";
    if (a.w_head_post) names[n++] = "k_head_mix";
    names[n++] = unfused_kernel_name(s, 3);
    return n;
}

// The launches follow unfused_chain(); each step reads maps[cur] and writes
// maps[cur ^ 1].  For the default composition that is logits -> map0,
// conv -> map1, softmax + mix -> map0, PV + GroupNorm from map0.  The exact
// indicator widens the logits and the first conv's halo by c_q - 1 keys.
mta_status launch_unfused(const mta_shape &s, const ForwardArgs &a, void *ws, cudaStream_t st,
                          const Trace &tr)
{
    float *maps[2] = {(float *)ws, (float *)ws + bh_tt(s)};
    const float *w_first = a.w_kq_3d ? a.w_kq_3d : a.w_kq;   // at most one is given
    const int band = (a.exact_mask && w_first) ? s.c_q - 1 : 0;
    int cur = 0, launch = 0;
    mta_status rc = MTA_OK;
    tr.before(launch, st);
    rc = logits(s, a.q, a.k, maps[0], band, st);
    tr.after(launch++, st);
    if (rc != MTA_OK) return rc;
    if (w_first) {
        tr.before(launch, st);
        launch_conv(s, maps[cur], maps[cur ^ 1], w_first, band, a.w_kq_3d ? s.c_h : 1, st);
        tr.after(launch++, st);
        cur ^= 1;
    }
    if (a.w_head_pre) {                           // mix of the logits, before the softmax
        tr.before(launch, st);
        rc = head_mix(s, maps[cur], maps[cur ^ 1], a.w_head_pre, st);
        tr.after(launch++, st);
        if (rc != MTA_OK) return rc;
        cur ^= 1;
    }
    tr.before(launch, st);
    rc = softmax_mix(s, maps[cur], maps[cur ^ 1], a.w_head, 0, st);
    tr.after(launch++, st);
    if (rc != MTA_OK) return rc;
    cur ^= 1;
    if (a.w_kq_post) {
        tr.before(launch, st);
        launch_conv(s, maps[cur], maps[cur ^ 1], a.w_kq_post, 0, 1, st);
        tr.after(launch++, st);
        cur ^= 1;
    }
    if (a.w_head_post) {
        tr.before(launch, st);
        rc = head_mix(s, maps[cur], maps[cur ^ 1], a.w_head_post, st);
        tr.after(launch++, st);
        if (rc != MTA_OK) return rc;
        cur ^= 1;
    }
    tr.before(launch, st);
    rc = pv_groupnorm(s, maps[cur], a, st);
    tr.after(launch, st);
    if (rc != MTA_OK) return rc;
    return cudaGetLastError() == cudaSuccess ? MTA_OK : MTA_ERR_CUDA;
}

mta_status launch_debug_attention(const mta_shape &s, const void *q, const void *k,
                                  const float *w_kq, const float *w_head, float *attn, int stage,
                                  void *ws, cudaStream_t st)
{
    float *map0 = (float *)ws;
    float *map1 = map0 + bh_tt(s);
    mta_status rc = logits(s, q, k, map0, 0, st);
    if (rc != MTA_OK) return rc;
    launch_conv(s, map0, map1, w_kq, 0, 1, st);
    rc = softmax_mix(s, map1, attn, w_head, stage == 0 ? 1 : 2, st);
    if (rc != MTA_OK) return rc;
    return cudaGetLastError() == cudaSuccess ? MTA_OK : MTA_ERR_CUDA;
}

}  // namespace mta
