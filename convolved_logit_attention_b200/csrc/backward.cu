// Backward pass of the MTA forward (the pages' default composition), on
// materialised T x T maps, all arithmetic in fp32 on CUDA cores.
//
// The pages give no backward pass ("Multi-Token Attention -- Paper Graph"
// reports training cost, Table 9, but prints no gradients); these are the
// gradients of the forward of section 3.4 -- Mask_0, the Eq. (4) key-query
// convolution, Mask_-inf, softmax, the Eq. (7) head mix after the softmax,
// A V, GroupNorm per head and the depth scale or the sigmoid gate -- by the
// chain rule, in reverse order of the steps:
//
//   recompute  A0 = Mask_0(Q K^T / sqrt d)                 -> M1
//              C = Conv_theta(A0)                           -> M2
//              P = softmax(C)                               -> M3
//              A = mix_w(P)                                 -> M2
//              O = A V                                      -> OD
//   k_gn_bwd   dO from dout through the affine GroupNorm and the scale;
//              partial sums of dgamma, dbeta (and dgate)    -> OD (in place)
//   k_causal_mm (transposed)  dV = A^T dO
//   logits_f32_io             dA = dO V^T (j <= i)         -> M2
//   k_mix_softmax_bwd  dP^{h'} = sum_h w[h][h'] dA^h, dw partials,
//              dC = P (dP - rowsum(dP P))                   -> M2 (in place)
//   k_conv_adj dA^ = Mask_0(Conv_theta^T(dC)): the adjoint stencil, taps
//              reading later queries and the mirrored keys  -> M3
//   k_dtheta   dtheta[i'][j'] partials: sum dC[i][j] A0[i-i'][j-j']
//   k_causal_mm dQ = dA^ K / sqrt d, (transposed) dK = dA^T Q / sqrt d
//   k_reduce   the partial sums, in a fixed order (deterministic)
//
// Only entries with key j <= query i of a map are written or read.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "io.cuh"
#include "tc_util.cuh"
#include "mta_internal.h"

namespace mta {
namespace {

constexpr int kMmRows = 64;      // k_causal_mm: 64 output rows x d
constexpr int kMmChunk = 32;     // contraction indices per staged chunk
constexpr int kMmAStride = kMmRows + 4;
constexpr int kMaxD = 128;
constexpr int kGnRows = 64;      // k_gn_bwd: query rows per CTA
constexpr int kAdjRows = 32;     // k_conv_adj / k_dtheta: 32 x 128 tiles
constexpr int kAdjCols = 128;
constexpr int kAdjStride = 164;  // halo row stride (floats), 4 (mod 32)
constexpr int kMaxCq = 8;

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// out[r][e] = scale * sum_c M[row(r)][col(c)] X[c][e] for one (b, h) and 64
// output rows, all d columns, fp32 out [B*H][T][d]:
//   kTrans = false: out row i, sum over keys j <= i of M[i][j] X[j]
//                   (O = A V, dQ = dA^ K / sqrt d)
//   kTrans = true:  out row j, sum over queries i >= j of M[i][j] X[i]
//                   (dV = A^T dO, dK = dA^T Q / sqrt d)
// Thread (warp w, lane l) accumulates rows 8w .. 8w+7 and columns 4l .. 4l+3.
// Each 32-index chunk of M is staged contraction-major, so a thread's 8 row
// values for one index are two 16-byte broadcast loads and its X values one
// 16-byte load.  The contraction runs in increasing index order.
template <typename TX, bool kTrans>
__global__ void __launch_bounds__(256)
k_causal_mm(const float *__restrict__ map, const TX *__restrict__ x, float *__restrict__ out,
            int T, int d, float scale)
{
    const int r0 = blockIdx.x * kMmRows;
    const size_t bh = blockIdx.y;
    __shared__ __align__(16) float asT[kMmChunk * kMmAStride];
    __shared__ __align__(16) float xs[kMmChunk * kMaxD];
    const int tid = threadIdx.x;
    const int rg = tid / 32, cg = (tid % 32) * 4;
    float acc[8][4];
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[u][w] = 0.f;
    const float *mb = map + bh * (size_t)T * T;
    const TX *xb = x + bh * (size_t)T * d;
    // contraction range: keys [0, min(T, r0 + 64)) or queries [r0, T)
    const int c_begin = kTrans ? r0 : 0;
    const int c_end = kTrans ? T : min(T, r0 + kMmRows);
    for (int c0 = c_begin; c0 < c_end; c0 += kMmChunk) {
        for (int idx = tid; idx < kMmRows * kMmChunk; idx += 256) {
            float val = 0.f;
            if (!kTrans) {   // row i = r0 + r, key j = c0 + c: coalesced along c
                const int r = idx / kMmChunk, c = idx % kMmChunk;
                const int i = r0 + r, j = c0 + c;
                if (i < T && j <= i) val = mb[(size_t)i * T + j];
                asT[c * kMmAStride + r] = val;
            } else {         // query i = c0 + c, key j = r0 + r: coalesced along r
                const int c = idx / kMmRows, r = idx % kMmRows;
                const int i = c0 + c, j = r0 + r;
                if (i < T && j < T && j <= i) val = mb[(size_t)i * T + j];
                asT[c * kMmAStride + r] = val;
            }
        }
        for (int r = tid / 32; r < kMmChunk; r += 8) {
            const int c = c0 + r;
            for (int e = (tid % 32) * 4; e < d; e += 128) {
                float y[4] = {0.f, 0.f, 0.f, 0.f};
                if (c < T) load4_f32(xb + (size_t)c * d + e, y);
#pragma unroll
                for (int u = 0; u < 4; ++u) xs[r * kMaxD + e + u] = y[u];
            }
        }
        __syncthreads();
        if (cg < d) {
#pragma unroll 4
            for (int c = 0; c < kMmChunk; ++c) {
                const float4 xa = *reinterpret_cast<const float4 *>(&asT[c * kMmAStride + rg * 8]);
                const float4 xb4 = *reinterpret_cast<const float4 *>(&asT[c * kMmAStride + rg * 8 + 4]);
                const float4 y = *reinterpret_cast<const float4 *>(&xs[c * kMaxD + cg]);
                const float a[8] = {xa.x, xa.y, xa.z, xa.w, xb4.x, xb4.y, xb4.z, xb4.w};
                const float yy[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
                for (int u = 0; u < 8; ++u)
#pragma unroll
                    for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(a[u], yy[w], acc[u][w]);
            }
        }
        __syncthreads();
    }
    if (cg < d) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int r = r0 + rg * 8 + u;
            if (r >= T) continue;
            float4 o = make_float4(acc[u][0] * scale, acc[u][1] * scale, acc[u][2] * scale,
                                   acc[u][3] * scale);
            *reinterpret_cast<float4 *>(out + (bh * T + r) * (size_t)d + cg) = o;
        }
    }
}

// GroupNorm + output scale backward for one (b, h) and 64 query rows.  With
// x^ = (O - mean) * rstd, y = gamma x^ + beta and out = s_h y (s_h the depth
// scale or sigmoid(g_h)):
//   dbeta_c  += s_h dout,   dgamma_c += s_h dout x^,
//   dg_h     += s_h (1 - s_h) sum dout y                  (gate only),
//   g_e = s_h dout_e gamma_e,
//   dO_e = rstd (g_e - mean_e(g) - x^_e mean_e(g x^)).
// Warp w takes rows 8w .. 8w+7, lane l the channels l, l+32, ...; OD holds O
// on entry and dO on exit.  Per-CTA partial sums go to
// pg/pb [B * nrb][H * d] and pgate [B * nrb][H] (row b * nrb + row block).
template <typename TIO>
__global__ void __launch_bounds__(256)
k_gn_bwd(float *__restrict__ od, const TIO *__restrict__ dout,
         const float *__restrict__ gn_weight, const float *__restrict__ gn_bias,
         float depth_scale, const float *__restrict__ gate, float eps, float *__restrict__ pg,
         float *__restrict__ pb, float *__restrict__ pgate, int T, int H, int d)
{
    const int rb = blockIdx.x, nrb = gridDim.x;
    const size_t bh = blockIdx.y;
    const int b = (int)(bh / H), h = (int)(bh % H);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    constexpr int KC = kMaxD / 32;                 // channels per lane at most
    __shared__ float red[8][2 * kMaxD + 1];
    const float s = gate ? 1.f / (1.f + expf(-gate[h])) : depth_scale;
    float accg[KC], accb[KC], accs = 0.f;
#pragma unroll
    for (int k = 0; k < KC; ++k) { accg[k] = 0.f; accb[k] = 0.f; }
    float gam[KC], bet[KC];
#pragma unroll
    for (int k = 0; k < KC; ++k) {
        const int e = lane + 32 * k;
        gam[k] = e < d ? gn_weight[h * d + e] : 0.f;
        bet[k] = e < d ? gn_bias[h * d + e] : 0.f;
    }
    for (int u = 0; u < kGnRows / 8; ++u) {
        const int t = rb * kGnRows + warp * (kGnRows / 8) + u;
        if (t >= T) break;
        float *orow = od + (bh * T + t) * (size_t)d;
        const TIO *drow = dout + ((size_t)b * T + t) * ((size_t)H * d) + (size_t)h * d;
        float o[KC], g[KC];
        float sum = 0.f;
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            const int e = lane + 32 * k;
            o[k] = e < d ? orow[e] : 0.f;
            g[k] = e < d ? to_f32(drow[e]) : 0.f;   // dout for now
            sum += o[k];
        }
        const float mean = warp_sum(sum) / d;
        float sq = 0.f;
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            const int e = lane + 32 * k;
            if (e < d) sq += (o[k] - mean) * (o[k] - mean);
        }
        const float rstd = 1.f / sqrtf(warp_sum(sq) / d + eps);
        float sg = 0.f, sgx = 0.f;
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            const int e = lane + 32 * k;
            if (e >= d) continue;
            const float xh = (o[k] - mean) * rstd;
            const float dy = s * g[k];                // d loss / d y
            accb[k] += dy;
            accg[k] += dy * xh;
            accs += g[k] * (gam[k] * xh + bet[k]);
            g[k] = dy * gam[k];                       // d loss / d x^
            o[k] = xh;
            sg += g[k];
            sgx += g[k] * xh;
        }
        const float mg = warp_sum(sg) / d, mgx = warp_sum(sgx) / d;
#pragma unroll
        for (int k = 0; k < KC; ++k) {
            const int e = lane + 32 * k;
            if (e < d) orow[e] = rstd * (g[k] - mg - o[k] * mgx);
        }
    }
    // partial sums of the CTA: warps through shared memory, fixed order
#pragma unroll
    for (int k = 0; k < KC; ++k) {
        const int e = lane + 32 * k;
        if (e < d) { red[warp][e] = accg[k]; red[warp][kMaxD + e] = accb[k]; }
    }
    accs = warp_sum(accs);
    if (lane == 0) red[warp][2 * kMaxD] = accs;
    __syncthreads();
    const size_t prow = (size_t)b * nrb + rb;
    for (int e = threadIdx.x; e < d; e += 256) {
        float a = 0.f, c = 0.f;
        for (int w = 0; w < 8; ++w) { a += red[w][e]; c += red[w][kMaxD + e]; }
        pg[prow * H * d + (size_t)h * d + e] = a;
        pb[prow * H * d + (size_t)h * d + e] = c;
    }
    if (threadIdx.x == 0 && pgate) {
        float a = 0.f;
        for (int w = 0; w < 8; ++w) a += red[w][2 * kMaxD];
        pgate[prow * H + h] = s * (1.f - s) * a;
    }
}

// Head-mix and softmax backward for one (b, group g, query row i):
//   dP^{h'}_j = sum_h w[h][h'] dA^h_j,
//   dw[h][h'] += sum_j dA^h_j P^{h'}_j   (partial per row: pw[g][b*T + i][h][h']),
//   dC^{h'}_j = P^{h'}_j (dP^{h'}_j - sum_j' dP^{h'}_j' P^{h'}_j'),
// over keys j <= i.  dA (in M2) is overwritten by dC; P is in M3.
template <int CH>
__global__ void __launch_bounds__(256)
k_mix_softmax_bwd(float *__restrict__ m2, const float *__restrict__ p3,
                  const float *__restrict__ w_head, float *__restrict__ pw, int B, int T, int H)
{
    const int i = blockIdx.x, bg = blockIdx.y;
    const int G = H / CH;
    const int b = bg / G, g = bg % G;
    __shared__ float wsm[CH * CH];
    __shared__ float red[8][CH * CH + CH];
    for (int idx = threadIdx.x; idx < CH * CH; idx += 256) wsm[idx] = w_head[(size_t)g * CH * CH + idx];
    __syncthreads();
    const size_t bh0 = (size_t)b * H + (size_t)g * CH;
    float dw[CH * CH], dot[CH];
#pragma unroll
    for (int x = 0; x < CH * CH; ++x) dw[x] = 0.f;
#pragma unroll
    for (int x = 0; x < CH; ++x) dot[x] = 0.f;
    for (int j = threadIdx.x; j <= i; j += 256) {
        float da[CH], p[CH];
#pragma unroll
        for (int hh = 0; hh < CH; ++hh) {
            const size_t off = ((bh0 + hh) * T + i) * (size_t)T + j;
            da[hh] = m2[off];
            p[hh] = p3[off];
        }
#pragma unroll
        for (int hi = 0; hi < CH; ++hi) {
            float dp = 0.f;
#pragma unroll
            for (int ho = 0; ho < CH; ++ho) {
                dp = fmaf(wsm[ho * CH + hi], da[ho], dp);
                dw[ho * CH + hi] = fmaf(da[ho], p[hi], dw[ho * CH + hi]);
            }
            dot[hi] = fmaf(dp, p[hi], dot[hi]);
        }
    }
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
#pragma unroll
    for (int x = 0; x < CH * CH; ++x) {
        const float v = warp_sum(dw[x]);
        if (lane == 0) red[warp][x] = v;
    }
#pragma unroll
    for (int x = 0; x < CH; ++x) {
        const float v = warp_sum(dot[x]);
        if (lane == 0) red[warp][CH * CH + x] = v;
    }
    __syncthreads();
    float rowdot[CH];
#pragma unroll
    for (int x = 0; x < CH; ++x) {
        float a = 0.f;
        for (int w = 0; w < 8; ++w) a += red[w][CH * CH + x];
        rowdot[x] = a;
    }
    if (threadIdx.x < CH * CH) {
        float a = 0.f;
        for (int w = 0; w < 8; ++w) a += red[w][threadIdx.x];
        pw[((size_t)g * B * T + (size_t)b * T + i) * (CH * CH) + threadIdx.x] = a;
    }
    // every thread has read its dA values above; the same thread rewrites them
    for (int j = threadIdx.x; j <= i; j += 256) {
        float da[CH], p[CH];
#pragma unroll
        for (int hh = 0; hh < CH; ++hh) {
            const size_t off = ((bh0 + hh) * T + i) * (size_t)T + j;
            da[hh] = m2[off];
            p[hh] = p3[off];
        }
#pragma unroll
        for (int hi = 0; hi < CH; ++hi) {
            float dp = 0.f;
#pragma unroll
            for (int ho = 0; ho < CH; ++ho) dp = fmaf(wsm[ho * CH + hi], da[ho], dp);
            m2[((bh0 + hi) * T + i) * (size_t)T + j] = p[hi] * (dp - rowdot[hi]);
        }
    }
}

// Halo fill of the stencil kernels.  The halo starts at the 16-byte group
// that holds key c0 (kOff = -LEFT mod 4 columns before it, c0 = -LEFT
// (mod 4)): tile[rr][x] = src[r0 + rr][c0 - kOff + x] for rr < rows,
// x < kLoadCols, zero where the row or column lies outside [0, T) or the key
// lies past the query (c > r).  With 16-byte rows (T % 4 == 0) every group
// is one cp.async copy, zero-filled when it lies outside (a group is wholly
// inside or outside [0, T)) or starts past the diagonal; in a tile whose
// halo reaches the diagonal the keys past it are cleared once the copies have
// landed.  The caller synchronises the CTA before reading the tile.
template <int kLoadCols, int kStride, int LEFT>
__device__ __forceinline__ void halo_fill(float *tile, const float *__restrict__ mb, int T,
                                          int rows, int r0, int c0)
{
    constexpr int kOff = ((-LEFT) % 4 + 4) % 4;
    static_assert(kLoadCols % 4 == 0, "whole groups");
    const int cbase = c0 - kOff;
    if ((T & 3) == 0) {
        constexpr int NQ = kLoadCols / 4;
        for (int idx = threadIdx.x; idx < rows * NQ; idx += blockDim.x) {
            const int rr = idx / NQ, qq = idx % NQ;
            const int r = r0 + rr, c = cbase + 4 * qq;
            const bool in = r >= 0 && r < T && c >= 0 && c < T && c <= r;
            tc::cp_async16(&tile[rr * kStride + 4 * qq], mb + (in ? (size_t)r * T + c : 0), in);
        }
        tc::cp_async_wait_all();
        if (cbase + kLoadCols - 1 > r0) {         // the halo reaches the diagonal
            __syncthreads();
            for (int idx = threadIdx.x; idx < rows * kLoadCols; idx += blockDim.x) {
                const int rr = idx / kLoadCols, x = idx % kLoadCols;
                if (cbase + x > r0 + rr) tile[rr * kStride + x] = 0.f;
            }
        }
    } else {
        for (int idx = threadIdx.x; idx < rows * kLoadCols; idx += blockDim.x) {
            const int rr = idx / kLoadCols, x = idx % kLoadCols;
            const int r = r0 + rr, c = cbase + x;
            tile[rr * kStride + x] =
                (r >= 0 && r < T && c >= 0 && c < T && c <= r) ? mb[(size_t)r * T + c] : 0.f;
        }
    }
}

// Adjoint of the Eq. (4) convolution with Mask_0 (the gradient of the raw
// logits): dst[r][c] = sum_{i'<c_q} sum_{j'} theta[i'][j'] dC[r+i'][c+j'] for
// c <= r, where dC is read as zero above the diagonal and outside [0,T)^2;
// dst is not written for c > r (no consumer reads there).  The 32 x 128
// output tile reads a (32 + c_q - 1)-row halo of dC below it; thread (warp w,
// lane l) owns output row l and columns 16w .. 16w+15, with the c_k taps
// applied from registers as in the forward k_conv.
template <int CK>
__global__ void __launch_bounds__(256, 4)
k_conv_adj(const float *__restrict__ src, float *__restrict__ dst, const float *__restrict__ w_kq,
           int T, int H, int c_q)
{
    constexpr int NC = kAdjCols / 8;
    constexpr int R = CK / 2;                     // keys reached to the left: j' >= -R
    constexpr int kOff = ((-R) % 4 + 4) % 4;      // the halo starts kOff keys before c0 - R
    constexpr int NV = (kOff + CK + NC - 1 + 3) / 4;
    constexpr int CKP = (CK + 3) / 4 * 4;
    constexpr int kLoadCols = 7 * NC + 4 * NV;
    static_assert(kLoadCols <= kAdjStride && kLoadCols >= kOff + kAdjCols + CK - 1, "halo width");
    const int r0 = blockIdx.y * kAdjRows, c0 = blockIdx.x * kAdjCols;
    if (c0 > r0 + kAdjRows - 1) return;           // tile entirely above the diagonal
    const size_t bh = blockIdx.z;
    const int h = (int)(bh % H);
    __shared__ __align__(16) float tile[(kAdjRows + kMaxCq - 1) * kAdjStride];
    __shared__ __align__(16) float th[kMaxCq * 16];
    const int tid = threadIdx.x;
    const int rows = kAdjRows + c_q - 1;
    const float *mb = src + bh * (size_t)T * T;
    halo_fill<kLoadCols, kAdjStride, R>(tile, mb, T, rows, r0, c0 - R);
    for (int idx = tid; idx < c_q * CKP; idx += 256) {
        const int ip = idx / CKP, jj = idx % CKP;
        th[idx] = jj < CK ? w_kq[((size_t)h * c_q + ip) * CK + jj] : 0.f;
    }
    __syncthreads();
    const int ro = tid % 32, cl = (tid / 32) * NC;
    float acc[NC];
#pragma unroll
    for (int u = 0; u < NC; ++u) acc[u] = 0.f;
    for (int ip = 0; ip < c_q; ++ip) {
        // output column c0 + cl + u, tap jj reads key c0 + cl + u - R + jj
        const float4 *seg4 = reinterpret_cast<const float4 *>(&tile[(ro + ip) * kAdjStride + cl]);
        float seg[4 * NV];
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            const float4 t = seg4[v];
            seg[4 * v] = t.x; seg[4 * v + 1] = t.y; seg[4 * v + 2] = t.z; seg[4 * v + 3] = t.w;
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
            for (int u = 0; u < NC; ++u) acc[u] = fmaf(tr[jj], seg[kOff + jj + u], acc[u]);
    }
    const int r = r0 + ro;
    if (r >= T) return;
    float *row = dst + bh * (size_t)T * T + (size_t)r * T;
#pragma unroll
    for (int g = 0; g < NC / 4; ++g) {
        const int cb = c0 + cl + 4 * g;
        if ((T & 3) == 0 && cb + 3 <= r) {       // 16-byte stores where the row segment is whole
            *reinterpret_cast<float4 *>(row + cb) =
                make_float4(acc[4 * g], acc[4 * g + 1], acc[4 * g + 2], acc[4 * g + 3]);
        } else {
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (cb + u <= r && cb + u < T) row[cb + u] = acc[4 * g + u];
        }
    }
}

// Partial sums of the kernel gradient over one 32 x 128 tile of outputs:
// part[tap] = sum_{(i, j) in tile, j <= i} dC[i][j] A0[i - i'][j - j'] for
// every tap (i', j'), with A0 read as Mask_0 and zero padding leave it (zero
// for c > r and outside [0,T)^2).  The same halo and thread layout as the
// forward k_conv; each query tap's c_k sums are reduced over the CTA (warp
// shuffles, then the 8 warps in fixed order) and written to
// part[(h * B*ntiles + b*ntiles + tile) * c_q*c_k + tap].
template <int CK>
__global__ void __launch_bounds__(256, 4)
k_dtheta(const float *__restrict__ dc, const float *__restrict__ a0, float *__restrict__ part,
         int B, int T, int H, int c_q)
{
    constexpr int NC = kAdjCols / 8;
    constexpr int L = (CK + 1) / 2 - 1;           // keys reached to the left by A0 taps
    constexpr int kOff = ((-L) % 4 + 4) % 4;      // the halo starts kOff keys before j0 - L
    constexpr int NV = (kOff + CK + NC - 1 + 3) / 4;
    constexpr int kLoadCols = 7 * NC + 4 * NV;
    static_assert(kLoadCols <= kAdjStride && kLoadCols >= kOff + kAdjCols + CK - 1, "halo width");
    const int nct = gridDim.x, nrt = gridDim.y;
    const int tile_id = blockIdx.y * nct + blockIdx.x;
    const int ntiles = nct * nrt;
    const int i0 = blockIdx.y * kAdjRows, j0 = blockIdx.x * kAdjCols;
    const size_t bh = blockIdx.z;
    const int b = (int)(bh / H), h = (int)(bh % H);
    float *dst = part + (((size_t)h * B + b) * ntiles + tile_id) * (size_t)(c_q * CK);
    if (j0 > i0 + kAdjRows - 1) {                 // above the diagonal: a zero partial
        for (int t = threadIdx.x; t < c_q * CK; t += 256) dst[t] = 0.f;
        return;
    }
    __shared__ __align__(16) float tile[(kAdjRows + kMaxCq - 1) * kAdjStride];
    __shared__ float red[2][8][16];           // double-buffered by query tap
    const int tid = threadIdx.x;
    const int rows = kAdjRows + c_q - 1;
    const float *mb = a0 + bh * (size_t)T * T;
    halo_fill<kLoadCols, kAdjStride, L>(tile, mb, T, rows, i0 - (c_q - 1), j0 - L);
    __syncthreads();
    const int ro = tid % 32, cl = (tid / 32) * NC;
    const int warp = tid / 32, lane = tid % 32;
    const int i = i0 + ro;
    float g[NC];
    {
        const float *grow = dc + bh * (size_t)T * T + (size_t)i * T;
#pragma unroll
        for (int q = 0; q < NC / 4; ++q) {
            const int jb = j0 + cl + 4 * q;
            if ((T & 3) == 0 && i < T && jb + 3 <= i) {   // 16-byte loads of whole segments
                const float4 t = *reinterpret_cast<const float4 *>(grow + jb);
                g[4 * q] = t.x; g[4 * q + 1] = t.y; g[4 * q + 2] = t.z; g[4 * q + 3] = t.w;
            } else {
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    g[4 * q + u] = (i < T && jb + u <= i) ? grow[jb + u] : 0.f;
            }
        }
    }
    for (int ip = 0; ip < c_q; ++ip) {
        const float4 *seg4 =
            reinterpret_cast<const float4 *>(&tile[(ro + c_q - 1 - ip) * kAdjStride + cl]);
        float seg[4 * NV];
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            const float4 t = seg4[v];
            seg[4 * v] = t.x; seg[4 * v + 1] = t.y; seg[4 * v + 2] = t.z; seg[4 * v + 3] = t.w;
        }
        float v[16];                              // the thread's partial of each key tap
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
            float a = 0.f;
            if (jj < CK) {
#pragma unroll
                for (int u = 0; u < NC; ++u) a = fmaf(g[u], seg[kOff + CK - 1 - jj + u], a);
            }
            v[jj] = a;
        }
        // Sum the 16 partials over the warp in 16 shuffles: at each step a lane
        // keeps the half of its values that its bit of the offset selects and
        // adds its partner's copy of that half; then lanes l and l ^ 1 both
        // hold the warp sum of tap k = (l >> 1) (a fixed order: deterministic).
#pragma unroll
        for (int o = 16, n = 16; o >= 2; o >>= 1, n >>= 1) {
            const bool hi = (lane & o) != 0;
#pragma unroll
            for (int x = 0; x < n / 2; ++x) {
                const float keep = hi ? v[x + n / 2] : v[x];
                const float send = hi ? v[x] : v[x + n / 2];
                v[x] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        }
        const float tap = v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
        const int k = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 +
                      ((lane >> 1) & 1);
        float (*rb)[16] = red[ip & 1];
        if ((lane & 1) == 0) rb[warp][k] = tap;
        __syncthreads();                          // red[ip & 1] is complete
        if (tid < CK) {
            float a = 0.f;
            for (int w = 0; w < 8; ++w) a += rb[w][tid];
            dst[ip * CK + tid] = a;
        }
    }
}

// out[o * n_inner + k] = sum over m < n_mid of part[(o * n_mid + m) * n_inner + k],
// one CTA per output element: strided partial sums, then a fixed-order tree.
__global__ void __launch_bounds__(256)
k_reduce(const float *__restrict__ part, float *__restrict__ out, int n_mid, int n_inner)
{
    const int o = blockIdx.y, k = blockIdx.x;
    __shared__ float red[256];
    float a = 0.f;
    for (int m = threadIdx.x; m < n_mid; m += 256)
        a += part[((size_t)o * n_mid + m) * n_inner + k];
    red[threadIdx.x] = a;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) out[(size_t)o * n_inner + k] = red[0];
}

struct BwdLayout {
    size_t m1, m2, m3, od, pg, pb, pgate, pw, pth, total;
    int nrb, ntiles;
};

size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

BwdLayout bwd_layout(const mta_shape &s)
{
    BwdLayout L;
    const size_t map = bh_tt(s) * sizeof(float);
    L.nrb = (s.T + kGnRows - 1) / kGnRows;
    L.ntiles = ((s.T + kAdjCols - 1) / kAdjCols) * ((s.T + kAdjRows - 1) / kAdjRows);
    size_t off = 0;
    L.m1 = off; off += al256(map);
    L.m2 = off; off += al256(map);
    L.m3 = off; off += al256(map);
    L.od = off; off += al256((size_t)s.B * s.H * s.T * s.d * sizeof(float));
    L.pg = off; off += al256((size_t)s.B * L.nrb * s.H * s.d * sizeof(float));
    L.pb = off; off += al256((size_t)s.B * L.nrb * s.H * s.d * sizeof(float));
    L.pgate = off; off += al256((size_t)s.B * L.nrb * s.H * sizeof(float));
    L.pw = off; off += al256((size_t)s.B * s.T * s.H * s.c_h * sizeof(float));   // G * B*T * c_h^2
    L.pth = off; off += al256((size_t)s.B * s.H * L.ntiles * s.c_q * s.c_k * sizeof(float));
    L.total = off;
    return L;
}

// k_mix_softmax_bwd with the row held in registers (T % 4 == 0, T <= 1024 NJ):
// thread t owns the 16-byte groups j = 4t + 1024n (n < NJ) of every head's
// dA and P row, read once; the reductions and the dC write use those
// registers.  Entries past the diagonal inside a group read as zero and are
// written as zero (nothing reads the map above the diagonal).
template <int CH, int NJ>
__global__ void __launch_bounds__(256)
k_mix_softmax_bwd_reg(float *__restrict__ m2, const float *__restrict__ p3,
                      const float *__restrict__ w_head, float *__restrict__ pw, int B, int T, int H)
{
    const int i = blockIdx.x, bg = blockIdx.y;
    const int G = H / CH;
    const int b = bg / G, g = bg % G;
    __shared__ float wsm[CH * CH];
    __shared__ float red[8][CH * CH + CH];
    for (int idx = threadIdx.x; idx < CH * CH; idx += 256) wsm[idx] = w_head[(size_t)g * CH * CH + idx];
    const size_t bh0 = (size_t)b * H + (size_t)g * CH;
    float da[NJ][CH][4], p[NJ][CH][4];
#pragma unroll
    for (int n = 0; n < NJ; ++n) {
        const int j4 = 4 * threadIdx.x + 1024 * n;
#pragma unroll
        for (int hh = 0; hh < CH; ++hh) {
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f), q = a;
            if (j4 <= i) {
                const size_t off = ((bh0 + hh) * T + i) * (size_t)T + j4;
                a = *reinterpret_cast<const float4 *>(m2 + off);
                q = *reinterpret_cast<const float4 *>(p3 + off);
            }
            const float av[4] = {a.x, a.y, a.z, a.w}, qv[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const bool live = j4 + e <= i;
                da[n][hh][e] = live ? av[e] : 0.f;
                p[n][hh][e] = live ? qv[e] : 0.f;
            }
        }
    }
    __syncthreads();                              // wsm
    float dw[CH * CH], dot[CH];
#pragma unroll
    for (int x = 0; x < CH * CH; ++x) dw[x] = 0.f;
#pragma unroll
    for (int x = 0; x < CH; ++x) dot[x] = 0.f;
#pragma unroll
    for (int n = 0; n < NJ; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e)
#pragma unroll
            for (int hi = 0; hi < CH; ++hi) {
                float dp = 0.f;
#pragma unroll
                for (int ho = 0; ho < CH; ++ho) {
                    dp = fmaf(wsm[ho * CH + hi], da[n][ho][e], dp);
                    dw[ho * CH + hi] = fmaf(da[n][ho][e], p[n][hi][e], dw[ho * CH + hi]);
                }
                dot[hi] = fmaf(dp, p[n][hi][e], dot[hi]);
            }
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
#pragma unroll
    for (int x = 0; x < CH * CH; ++x) {
        const float v = warp_sum(dw[x]);
        if (lane == 0) red[warp][x] = v;
    }
#pragma unroll
    for (int x = 0; x < CH; ++x) {
        const float v = warp_sum(dot[x]);
        if (lane == 0) red[warp][CH * CH + x] = v;
    }
    __syncthreads();
    float rowdot[CH];
#pragma unroll
    for (int x = 0; x < CH; ++x) {
        float a = 0.f;
        for (int w = 0; w < 8; ++w) a += red[w][CH * CH + x];
        rowdot[x] = a;
    }
    if (threadIdx.x < CH * CH) {
        float a = 0.f;
        for (int w = 0; w < 8; ++w) a += red[w][threadIdx.x];
        pw[((size_t)g * B * T + (size_t)b * T + i) * (CH * CH) + threadIdx.x] = a;
    }
#pragma unroll
    for (int n = 0; n < NJ; ++n) {
        const int j4 = 4 * threadIdx.x + 1024 * n;
        if (j4 > i) continue;
#pragma unroll
        for (int hi = 0; hi < CH; ++hi) {
            float o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float dp = 0.f;
#pragma unroll
                for (int ho = 0; ho < CH; ++ho) dp = fmaf(wsm[ho * CH + hi], da[n][ho][e], dp);
                o[e] = p[n][hi][e] * (dp - rowdot[hi]);
            }
            *reinterpret_cast<float4 *>(m2 + ((bh0 + hi) * T + i) * (size_t)T + j4) =
                make_float4(o[0], o[1], o[2], o[3]);
        }
    }
}

template <int CH>
void launch_mix_softmax_bwd(const mta_shape &s, float *m2, const float *p3, const float *w,
                            float *pw, cudaStream_t st)
{
    const dim3 grid(s.T, s.B * (s.H / CH));
    if constexpr (CH <= 2) {
        if (s.T % 4 == 0 && s.T <= 4096) {       // the row fits the registers of one CTA
            switch ((s.T + 1023) / 1024) {
                case 1: k_mix_softmax_bwd_reg<CH, 1><<<grid, 256, 0, st>>>(m2, p3, w, pw, s.B, s.T, s.H); return;
                case 2: k_mix_softmax_bwd_reg<CH, 2><<<grid, 256, 0, st>>>(m2, p3, w, pw, s.B, s.T, s.H); return;
                case 3: k_mix_softmax_bwd_reg<CH, 3><<<grid, 256, 0, st>>>(m2, p3, w, pw, s.B, s.T, s.H); return;
                default: k_mix_softmax_bwd_reg<CH, 4><<<grid, 256, 0, st>>>(m2, p3, w, pw, s.B, s.T, s.H); return;
            }
        }
    }
    k_mix_softmax_bwd<CH><<<grid, 256, 0, st>>>(m2, p3, w, pw, s.B, s.T, s.H);
}

mta_status mix_softmax_bwd(const mta_shape &s, float *m2, const float *p3, const float *w,
                           float *pw, cudaStream_t st)
{
    switch (s.c_h) {
        case 1: launch_mix_softmax_bwd<1>(s, m2, p3, w, pw, st); break;
        case 2: launch_mix_softmax_bwd<2>(s, m2, p3, w, pw, st); break;
        case 4: launch_mix_softmax_bwd<4>(s, m2, p3, w, pw, st); break;
        case 8: launch_mix_softmax_bwd<8>(s, m2, p3, w, pw, st); break;
        case 16: launch_mix_softmax_bwd<16>(s, m2, p3, w, pw, st); break;
        default: return MTA_ERR_UNSUPPORTED;
    }
    return MTA_OK;
}

void conv_adj_and_dtheta(const mta_shape &s, const float *dc, const float *a0, float *dst,
                         float *pth, const float *w_kq, cudaStream_t st, const Trace &tr,
                         int launch)
{
    dim3 g((s.T + kAdjCols - 1) / kAdjCols, (s.T + kAdjRows - 1) / kAdjRows, s.B * s.H);
    switch (s.c_k) {
#define MTA_ADJ_CASE(n)                                                                         \
        case n:                                                                                 \
            tr.before(launch, st);                                                              \
            k_conv_adj<n><<<g, 256, 0, st>>>(dc, dst, w_kq, s.T, s.H, s.c_q);                   \
            tr.after(launch, st);                                                               \
            tr.before(launch + 1, st);                                                          \
            k_dtheta<n><<<g, 256, 0, st>>>(dc, a0, pth, s.B, s.T, s.H, s.c_q);                  \
            tr.after(launch + 1, st);                                                           \
            break;
        MTA_ADJ_CASE(1) MTA_ADJ_CASE(2) MTA_ADJ_CASE(3) MTA_ADJ_CASE(4) MTA_ADJ_CASE(5)
        MTA_ADJ_CASE(6) MTA_ADJ_CASE(7) MTA_ADJ_CASE(8) MTA_ADJ_CASE(9) MTA_ADJ_CASE(10)
        MTA_ADJ_CASE(11) MTA_ADJ_CASE(12) MTA_ADJ_CASE(13) MTA_ADJ_CASE(14) MTA_ADJ_CASE(15)
#undef MTA_ADJ_CASE
        default: break;   // c_k <= 15 is checked before any launch
    }
}

template <bool kTrans>
mta_status causal_mm(const mta_shape &s, const float *map, const void *x, bool x_io, float *out,
                     float scale, cudaStream_t st)
{
    if (mm_tf32_supported(s)) return causal_mm_tf32(s, kTrans, map, x, x_io, out, scale, st);
    dim3 g((s.T + kMmRows - 1) / kMmRows, s.B * s.H);
    if (x_io && s.io == MTA_BF16)
        k_causal_mm<__nv_bfloat16, kTrans><<<g, 256, 0, st>>>(map, (const __nv_bfloat16 *)x, out,
                                                              s.T, s.d, scale);
    else
        k_causal_mm<float, kTrans><<<g, 256, 0, st>>>(map, (const float *)x, out, s.T, s.d,
                                                      scale);
    return MTA_OK;
}

void reduce(const float *part, float *out, int n_outer, int n_mid, int n_inner, cudaStream_t st)
{
    k_reduce<<<dim3(n_inner, n_outer), 256, 0, st>>>(part, out, n_mid, n_inner);
}

}  // namespace

const char *backward_kernel_name(const mta_shape &s, int index)
{
    static const char *const names[kBackwardKernels] = {
        "k_logits", "k_conv", "k_softmax_mix", "k_head_mix", "k_causal_mm", "k_gn_bwd",
        "k_causal_mm", "k_logits", "k_mix_softmax_bwd", "k_conv_adj", "k_dtheta", "k_causal_mm",
        "k_causal_mm", "k_reduce"};
    if (index < 0 || index >= kBackwardKernels) return nullptr;
    // the recomputed logits take the chain's kernel for the shape; at d = 64
    // or 128 the fp32 products (A V, dV, dA, dQ, dK) run as 3xTF32 MMAs
    if (index == 0) return unfused_kernel_name(s, 0);
    if (mm_tf32_supported(s) && (index == 4 || index == 6 || index == 7 || index == 11 ||
                                 index == 12))
        return "k_mm_tf32";
    return names[index];
}

size_t backward_workspace_bytes(const mta_shape &s) { return bwd_layout(s).total; }

mta_status launch_backward(const mta_shape &s, const ForwardArgs &a, const BackwardArgs &g,
                           void *ws, cudaStream_t st, const Trace &tr)
{
    const BwdLayout L = bwd_layout(s);
    uint8_t *w = (uint8_t *)ws;
    float *m1 = (float *)(w + L.m1), *m2 = (float *)(w + L.m2), *m3 = (float *)(w + L.m3);
    float *od = (float *)(w + L.od);
    float *pg = (float *)(w + L.pg), *pb = (float *)(w + L.pb), *pgate = (float *)(w + L.pgate);
    float *pw = (float *)(w + L.pw), *pth = (float *)(w + L.pth);
    const float rsd = 1.0f / sqrtf((float)s.d);
    mta_status rc = MTA_OK;
    int n = 0;
    // forward recompute
    tr.before(n, st); rc = logits(s, a.q, a.k, m1, 0, st); tr.after(n++, st);
    if (rc != MTA_OK) return rc;
    tr.before(n, st); launch_conv(s, m1, m2, a.w_kq, 0, 1, st); tr.after(n++, st);
    tr.before(n, st); rc = softmax_mix(s, m2, m3, nullptr, 0, st); tr.after(n++, st);
    if (rc != MTA_OK) return rc;
    tr.before(n, st); rc = head_mix(s, m3, m2, a.w_head, st); tr.after(n++, st);
    if (rc != MTA_OK) return rc;
    tr.before(n, st); rc = causal_mm<false>(s, m2, a.v, true, od, 1.f, st); tr.after(n++, st);
    if (rc != MTA_OK) return rc;
    // GroupNorm and output scale
    tr.before(n, st);
    {
        dim3 grid(L.nrb, s.B * s.H);
        if (s.io == MTA_BF16)
            k_gn_bwd<__nv_bfloat16><<<grid, 256, 0, st>>>(
                od, (const __nv_bfloat16 *)g.dout, a.gn_weight, a.gn_bias, a.depth_scale, a.gate,
                s.gn_eps, pg, pb, a.gate ? pgate : nullptr, s.T, s.H, s.d);
        else
            k_gn_bwd<float><<<grid, 256, 0, st>>>(od, (const float *)g.dout, a.gn_weight,
                                                  a.gn_bias, a.depth_scale, a.gate, s.gn_eps, pg,
                                                  pb, a.gate ? pgate : nullptr, s.T, s.H, s.d);
    }
    tr.after(n++, st);
    // dV = A^T dO, then dA = dO V^T over the A map
    tr.before(n, st); rc = causal_mm<true>(s, m2, od, false, g.dv, 1.f, st); tr.after(n++, st);
    if (rc != MTA_OK) return rc;
    tr.before(n, st);
    if (mm_tf32_supported(s)) rc = logits_f32_tf32(s, od, a.v, 1.f, m2, st);
    else logits_f32_io(s, od, a.v, 1.f, m2, st);
    tr.after(n++, st);
    if (rc != MTA_OK) return rc;
    // head mix and softmax: dA -> dC in M2, dw partials
    tr.before(n, st); rc = mix_softmax_bwd(s, m2, m3, a.w_head, pw, st); tr.after(n++, st);
    if (rc != MTA_OK) return rc;
    // convolution: dA^ in M3 (P is dead), dtheta partials from dC and A0
    conv_adj_and_dtheta(s, m2, m1, m3, pth, a.w_kq, st, tr, n);
    n += 2;
    // dQ = dA^ K / sqrt d, dK = dA^T Q / sqrt d
    tr.before(n, st); rc = causal_mm<false>(s, m3, a.k, true, g.dq, rsd, st); tr.after(n++, st);
    if (rc != MTA_OK) return rc;
    tr.before(n, st); rc = causal_mm<true>(s, m3, a.q, true, g.dk, rsd, st); tr.after(n++, st);
    if (rc != MTA_OK) return rc;
    // the parameter gradients
    tr.before(n, st);
    const int G = s.H / s.c_h;
    reduce(pg, g.dgn_weight, 1, s.B * L.nrb, s.H * s.d, st);
    reduce(pb, g.dgn_bias, 1, s.B * L.nrb, s.H * s.d, st);
    if (a.gate) reduce(pgate, g.dgate, 1, s.B * L.nrb, s.H, st);
    reduce(pw, g.dw_head, G, s.B * s.T, s.c_h * s.c_h, st);
    reduce(pth, g.dw_kq, s.H, s.B * L.ntiles, s.c_q * s.c_k, st);
    tr.after(n, st);
    return cudaGetLastError() == cudaSuccess ? MTA_OK : MTA_ERR_CUDA;
}

}  // namespace mta
