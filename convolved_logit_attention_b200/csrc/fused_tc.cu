// Fused MTA forward on sm_100a tensor cores (bf16 operands, fp32 accumulate).
//
// The key-query convolution of "Multi-Token Attention -- Paper Graph",
// section 3.4, Eq. (4)/(5), is linear in the logits, so away from the
// diagonal it folds into the contraction:
//     C[i][j] = sum_{i'} q_{i-i'} . Kf^{(i')}_j,
//     Kf^{(i')}_j = sum_{j'} theta[i'][j'] k_{j-j'} / sqrt(d)
// (q rows before the sequence and k rows outside it are zero).  The first
// mask of Eq. (5) zeroes logits of future keys before the convolution; the
// fold includes those terms for pairs (i, j) within D_m = c_q - 1 +
// floor(c_k/2) diagonals of the main one, and a per-row correction table
// subtracts them there.
//
// Three kernels, launched back to back on the caller's stream (the last two
// with programmatic dependent launch, so each is scheduled while its
// predecessor drains):
//   k_fold           the prologue, CTAs in two roles:
//                    - per (b, h, 128-key block): Kf^{(i')} for every i' (fp16,
//                      scaled by log2(e)/sqrt(d) so that the softmax runs on
//                      exp2).  fp16 carries three more mantissa bits than bf16
//                      for the folded logits; values outside its range raise an
//                      error.
//                    - per (b, h, 64-row half block): the query rows (fp16) in
//                      the permuted order the main kernel's shifted operand
//                      needs, and the correction table corr[i][e] for key
//                      j = i - e.
//   k_mta_fused      per (b, source head h', 128 query rows): for every key
//                    tile, S = sum_{i'} Q_{shift i'} Kf^{(i')T} on tcgen05
//                    (TMEM accumulator), correction + causal mask + online
//                    softmax on CUDA cores, then U^{h,h'} += P~ V^h for every
//                    head h of the group (post-softmax head mixing, Eq. (7),
//                    with per-source-head normalisation deferred to the end).
//                    Writes (w[h][h'] / l^{h'}) U^{h,h'} per row, in fp16.
//   k_mix_groupnorm  per (b, query row): O^h = sum_{h'} of those partials,
//                    per-head GroupNorm with warp-shuffle reductions, depth
//                    scale, bf16 store.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "mta_internal.h"
#include "tc_util.cuh"
#include "tmap.h"

namespace mta {
namespace {

constexpr int kBM = 128;          // query rows per CTA (TMEM lanes)
constexpr int kBN = 128;          // keys per tile
constexpr int kCorrW = 16;        // correction entries stored per row (D_m <= 14); must be 16
static_assert(kCorrW == 16, "band tiles index the table modulo 16");
constexpr int kCorrStride = 17;   // shared-memory row stride of that table (conflict-free reads)
constexpr int kScrStride = 36;    // floats per scratch row: 16-B aligned, conflict-free by float4
constexpr float kLog2e = 1.4426950408889634f;
// Named barriers at which the MMA issuer meets its gate warp: one per ring
// slot and one for the Q tile.
constexpr int kGateStage0 = 1;     // ids 1 .. kStages (at most 8)
constexpr int kGateQ = 9;
constexpr long long kWaitBudget = 1ll << 30;   // ~0.55 s at 1.965 GHz per wait

// Device error word: bit 0 a bounded wait expired, bit 1 a folded operand
// fell outside the fp16 range.
__device__ unsigned int g_fused_error;
constexpr unsigned int kErrTimeout = 1u, kErrRange = 2u;

// Rows of the permuted query block: NA atoms of 8 rows; atom a, row s holds
// query i0 - (c_q - 1) + a + 16 s.
__host__ __device__ inline int q_atoms(int c_q) { return 16 + c_q - 1; }
__host__ __device__ inline int d_m(int c_q, int c_k) { return c_q - 1 + c_k / 2; }

// ------------------------------------------------------------ prologue

constexpr int kProRows = 128;     // rows (keys and queries) per prologue CTA
constexpr int kProQLo = 7;        // query rows before the block whose future logits are needed
constexpr int kAuxRows = 64;      // query rows per aux prologue CTA
constexpr int kProThreads = 256;  // threads of a prologue CTA (either role)

// Packed fp32 pairs (Blackwell's f32x2 arithmetic): one instruction does two
// fp32 FMAs, each rounded once, exactly as fmaf would.
__device__ __forceinline__ unsigned long long f2_pack(float lo, float hi)
{
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 f2_unpack(unsigned long long v)
{
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
    return make_float2(lo, hi);
}
__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b,
                                                     unsigned long long c)
{
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
// A bf16 pair as a packed fp32 pair (widening is exact).
__device__ __forceinline__ unsigned long long bf2_to_f2(uint32_t v)
{
    return f2_pack(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}

// Warp-level bf16 MMA (m16n8k16, fp32 accumulate) and its shared-memory
// fragment loads, for the small banded product of the aux prologue.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void *p)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(tc::smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x2(uint32_t (&r)[2], const void *p)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
                 : "=r"(r[0]), "=r"(r[1])
                 : "r"(tc::smem_u32(p)));
}
__device__ __forceinline__ void mma_16816_bf16(float (&d)[4], const uint32_t (&a)[4],
                                               const uint32_t (&b)[2])
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
                 "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Largest value of m over the CTA (blockDim.x a multiple of 32, at most
// 256); every thread gets the result.  `red` is 8 floats of shared memory.
__device__ float block_max(float m, float *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __syncthreads();                           // red may still be read by an earlier use
    if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = m;
    __syncthreads();
    float r = red[0];
    for (int w = 1; w < (int)blockDim.x / 32; ++w) r = fmaxf(r, red[w]);
    return r;
}

// The largest |x| bit pattern of each bf16 half of v, folded into the two
// halfword lanes of m (|x| orders like its bits with the sign cleared).
__device__ __forceinline__ uint32_t absmax_bits(uint32_t m, uint32_t v)
{
    uint32_t r;
    asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(m), "r"(v & 0x7fff7fffu));
    return r;
}
// The float value of the larger lane; +inf when it is a NaN or infinity.
__device__ __forceinline__ float bits_to_absmax(uint32_t m)
{
    const uint32_t top = max(m & 0xffffu, m >> 16);
    return top >= 0x7f80u ? INFINITY : __uint_as_float(top << 16);
}

// The power-of-two exponent e >= 0 of a block's fp16 operand scale, from the
// largest |value| of the block: 0 when it fits fp16 (the usual case: the
// block is then computed exactly as without scaling), else the smallest e
// with max * 2^-e <= 2^15.  -1 for a non-finite max.
__device__ __forceinline__ int range_exponent(float mx)
{
    if (mx <= 65504.f) return 0;
    if (!(mx <= 3.0e38f)) return -1;
    int e = 0;
    frexpf(mx / 32768.f, &e);                  // mx / 2^15 <= 2^e
    return e;
}

// Folded keys of one 128-key block with the taps in ths (the logit scale,
// and a range scale if any, included): thread = one column pair x a run of
// RPG consecutive keys, in windows of SUB keys.  Kf^{(i')}_j =
// sum_jj ths[i'][jj] k_{j + RT - jj}, with the taps zero-padded to CK (CK =
// c_k for the common sizes, 15 otherwise) and centred like the real kernel,
// so every tap index is a compile-time constant.  The two columns of a pair
// share every tap: one packed f32x2 FMA per tap.  Returns the largest |Kf|
// this thread wrote (after the fp16 rounding: +inf where a value overflowed).
template <int D, int CK>
__device__ __forceinline__ float fold_keys_run(int blk, int bh, const __nv_bfloat16 *__restrict__ k,
                                               const float *ths, __half *__restrict__ kf, int T,
                                               int Tp, int c_q)
{
    constexpr int EP = D / 2;                  // column pairs
    constexpr int RG = 256 / EP;               // key runs per block
    constexpr int RPG = kProRows / RG;         // keys per run
    constexpr int RT = CK / 2, LT = CK - 1 - RT;
    constexpr int SUB = 16;
    constexpr int WS = SUB + CK - 1;           // window rows
    const int j0 = blk * kProRows;
    const int ep = threadIdx.x % EP, rg = threadIdx.x / EP;
    const __nv_bfloat16 *kh = k + (size_t)bh * T * D + 2 * ep;
    __half2 amax = __floats2half2_rn(0.f, 0.f);
#pragma unroll 1
    for (int sub = 0; sub < RPG / SUB; ++sub) {
        const int jr0 = j0 + rg * RPG + sub * SUB;     // first key of the window
        unsigned long long win[WS];
#pragma unroll
        for (int w = 0; w < WS; ++w) {
            const int row = jr0 - LT + w;
            const uint32_t v = (row >= 0 && row < T) ? *(const uint32_t *)(kh + (size_t)row * D) : 0u;
            win[w] = bf2_to_f2(v);
        }
        for (int ip = 0; ip < c_q; ++ip) {
            unsigned long long tt[CK];
#pragma unroll
            for (int jj = 0; jj < CK; ++jj) {
                const float t = ths[ip * CK + jj];
                tt[jj] = f2_pack(t, t);
            }
            __half *dst = kf + (((size_t)bh * c_q + ip) * Tp + jr0) * D + 2 * ep;
#pragma unroll
            for (int r = 0; r < SUB; ++r) {
                unsigned long long acc = 0ull;
#pragma unroll
                for (int jj = 0; jj < CK; ++jj) acc = f2_fma(tt[jj], win[r + CK - 1 - jj], acc);
                const float2 a = f2_unpack(acc);
                const __half2 hv = __floats2half2_rn(a.x, a.y);
                amax = __hmax2(amax, __habs2(hv));
                *(__half2 *)(dst + (size_t)r * D) = hv;
            }
        }
    }
    const float2 am = __half22float2(amax);
    return fmaxf(am.x, am.y);
}

// Largest |x| over rows [r_lo, r_hi) (clipped to [0, T)) of one head's bf16
// [T][D] rows, over the CTA (every thread gets it; +inf for a non-finite
// element).  `red` is 8 floats of shared memory.
template <int D>
__device__ float rows_absmax(const __nv_bfloat16 *__restrict__ head, int r_lo, int r_hi, int T,
                             float *red)
{
    const int lo = r_lo > 0 ? r_lo : 0, hi = r_hi < T ? r_hi : T;
    uint32_t mb = 0u;
    for (int idx = threadIdx.x; idx < (hi - lo) * (D / 8); idx += blockDim.x) {
        const uint4 v = *(const uint4 *)(head + (size_t)(lo + idx / (D / 8)) * D + 8 * (idx % (D / 8)));
        mb = absmax_bits(absmax_bits(absmax_bits(absmax_bits(mb, v.x), v.y), v.z), v.w);
    }
    return block_max(bits_to_absmax(mb), red);
}

// Folded keys: one CTA per (128-key block, b*H + h), 256 threads.  The
// block is written as computed, and an fp16 overflow shows up as +inf in the
// largest |Kf| written.  Such a block (a bf16 input of order 1e4 or more) is
// computed a second time with the taps scaled by 2^-e, exactly, e chosen from
// the bound max |k| over the window times max_{i'} sum_{j'} |tap|; the main
// kernel multiplies the logits of this key block back by 2^e.
template <int D, int CK>
__device__ __forceinline__ void fold_keys_block(int blk, int bh, const __nv_bfloat16 *__restrict__ k,
                                                const float *__restrict__ w_kq,
                                                __half *__restrict__ kf, int *__restrict__ kexp,
                                                int T, int Tp, int H, int nqb, int c_q, int c_k,
                                                float scale)
{
    constexpr int RT = CK / 2;
    __shared__ float ths[8 * CK];              // zero-padded taps times the logit scale
    __shared__ float red[8];
    const int h = bh % H;
    const int tid = threadIdx.x;
    const int R = c_k / 2, shift = RT - R;     // real tap jj sits at padded index jj + shift
    for (int idx = tid; idx < 8 * CK; idx += 256) {
        const int ip = idx / CK, jp = idx % CK - shift;
        ths[idx] = (ip < c_q && jp >= 0 && jp < c_k) ? w_kq[((size_t)h * c_q + ip) * c_k + jp] * scale
                                                     : 0.f;
    }
    __syncthreads();
    const float amax = fold_keys_run<D, CK>(blk, bh, k, ths, kf, T, Tp, c_q);
    int e = 0;
    if (block_max(amax, red) > 65504.f) {      // the same in every thread; rare
        constexpr int LT = CK - 1 - RT;
        const int j0 = blk * kProRows;
        const float mk = rows_absmax<D>(k + (size_t)bh * T * D, j0 - LT, j0 + kProRows + RT, T, red);
        float tb = 0.f;
        for (int ip = 0; ip < c_q; ++ip) {
            float a = 0.f;
            for (int jj = 0; jj < CK; ++jj) a += fabsf(ths[ip * CK + jj]);
            tb = fmaxf(tb, a);
        }
        e = range_exponent(mk * tb);
        // reported either way: a non-finite input, or a block beyond fp16 that
        // stays finite but whose logits near the diagonal lose accuracy
        if (tid == 0) atomicOr(&g_fused_error, kErrRange);
        if (e < 0) {
            e = 0;
        } else {
            __syncthreads();                   // every thread has read the taps
            for (int idx = tid; idx < 8 * CK; idx += 256) ths[idx] = ldexpf(ths[idx], -e);
            __syncthreads();
            fold_keys_run<D, CK>(blk, bh, k, ths, kf, T, Tp, c_q);
        }
    }
    if (tid == 0) kexp[(size_t)bh * nqb + blk] = e;
}

// The terms of four correction entries e = E0 .. E0+3 of one row: for every
// query tap i' < c_q and padded key tap jj, thp[i'][jj] times the future logit
// F[i - i'][delta] (frow0 is row i's F row; row i - i' lies i' rows of
// stride fstride before it), delta = i' + RT - jj - e.  Every index is static
// after unrolling, so terms outside 1 <= delta <= 14 are never emitted.
template <int CK, int E0, bool EXACT>
__device__ __forceinline__ void corr_terms(float (&acc)[4], const float *frow0, int fstride,
                                           const float *thp, int c_q)
{
    constexpr int RT = CK / 2;
#pragma unroll
    for (int ip = 0; ip < 8; ++ip) {
        if (ip < c_q) {
            const float *frow = frow0 - ip * fstride;
#pragma unroll
            for (int jj = 0; jj < CK; ++jj) {
                if (ip + RT - jj - E0 < 1) continue;          // every delta of this tap < 1
                const float t = thp[ip * CK + jj];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int delta = ip + RT - jj - (E0 + e);
                    if (delta >= 1 && delta <= kCorrW - 2) {
                        const float f = (EXACT && delta <= ip) ? 0.f : frow[delta - 1];
                        acc[e] = fmaf(t, f, acc[e]);
                    }
                }
            }
        }
    }
}

// The rest of the prologue: one CTA per (64-row block, b*H + h), 256
// threads, three sections:
//  (b) the block's query rows in the permuted atom order, converted to fp16.
//  (c) future logits F[r][delta] = scale * q_r . k_{r+delta}, delta in
//      [1, D_m], for r in [j0 - 7, j0 + 64), from shared-memory copies of
//      the rows involved.
//  (d) corr[i][e] = sum over taps (i', j') with delta = i' - j' - e >= 1 and
//      r = i - i' >= 0 of theta[i'][j'] F[r][delta]: the terms of keys past
//      the tap's own query row r, which Mask_0 of Eq. (5) removes.  With
//      `exact` (the indicator of Eq. (4), which keeps a tap whenever its key
//      is not past the output's query i) only the terms with delta > i',
//      that is key r + delta > i, are removed.  EXACT is that flag, a template
//      parameter so that the common path carries no per-term select.
template <int D, int CK, bool EXACT>
__device__ __forceinline__ void fold_aux_block(int blk, int bh, const __nv_bfloat16 *__restrict__ q,
                                               const __nv_bfloat16 *__restrict__ k,
                                               const float *__restrict__ w_kq,
                                               __half *__restrict__ qp, float *__restrict__ corr,
                                               int *__restrict__ qexp, int T, int Tp, int H,
                                               int nqb, int c_q, int c_k, float scale)
{
    constexpr int QR = kProQLo + kAuxRows;
    constexpr int RT = CK / 2;                 // the taps' padded centre
    constexpr int kFs = kCorrW + 1;            // F row stride: rows of a warp hit distinct banks
    __shared__ float thp[8 * CK];              // taps zero-padded to CK and centred at RT
    __shared__ float fs[QR * kFs];
    extern __shared__ __align__(16) __nv_bfloat16 qk_sm[];   // section (c) row copies
    const int h = bh % H;
    const int j0 = blk * kAuxRows;
    // the 128-row query block whose permuted rows this CTA writes one half of
    const int qblk = j0 / kProRows, half = (j0 % kProRows) / kAuxRows;
    const int tid = threadIdx.x;
    const size_t head_off = (size_t)bh * T * D;
    const int shift = RT - c_k / 2;            // real tap jj sits at padded index jj + shift
    for (int idx = tid; idx < 8 * CK; idx += kProThreads) {
        const int ip = idx / CK, jj = idx % CK - shift;
        thp[idx] = (ip < c_q && jj >= 0 && jj < c_k) ? w_kq[((size_t)h * c_q + ip) * c_k + jj] : 0.f;
    }
    // Row copies in shared memory, all in flight at once (cp.async): q rows
    // [j0-7, j0+64) and k rows [j0-6, j0+78), zero outside [0, T); rows are
    // padded by 16 bytes so that threads on different rows hit different banks,
    // and both copies are padded with zero rows to whole MMA tiles (QRP, KRP).
    constexpr int RS = D + 8;                  // padded row stride in bf16 elements
    constexpr int KR = QR + kCorrW - 3;        // k rows j0-6 .. j0+77 (r + delta <= j0+63+14)
    constexpr int QRP = (QR + 15) / 16 * 16;   // 80 q rows: five 16-row MMA tiles
    constexpr int KRP = QRP + 16;              // 96 k rows: each tile reaches 32 rows on
    constexpr int CPR = D / 8;                 // 16-byte chunks per row
    __nv_bfloat16 *qsm = qk_sm;                // [QRP][RS]
    __nv_bfloat16 *ksm = qk_sm + QRP * RS;     // [KRP][RS]
    constexpr int RP = kProThreads / CPR;      // rows per pass of the CTA
    static_assert(kProThreads % CPR == 0, "whole rows per pass");
    const int c8 = tid % CPR;                  // the thread's 16-byte chunk of every row
    for (int lr = tid / CPR; lr < QRP; lr += RP) {
        const int g = j0 - kProQLo + lr;
        const bool in = lr < QR && g >= 0 && g < T;
        tc::cp_async16(qsm + lr * RS + 8 * c8, q + head_off + (size_t)(in ? g : 0) * D + 8 * c8, in);
    }
    for (int lr = tid / CPR; lr < KRP; lr += RP) {
        const int g = j0 - (kProQLo - 1) + lr;
        const bool in = lr < KR && g >= 0 && g < T;
        tc::cp_async16(ksm + lr * RS + 8 * c8, k + head_off + (size_t)(in ? g : 0) * D + 8 * c8, in);
    }
    // Range of the 128-row block's permuted queries: both halves' CTAs take
    // the largest |q| over the rows [i0 - 7, i0 + 128), their own 71 rows from
    // the copy and the other half's 64 rows loaded here, while the copy is in
    // flight.  A block beyond the fp16 range is scaled by 2^-e before the
    // rounding, and the main kernel multiplies its logits back by 2^e.
    const int i0 = qblk * kProRows;
    constexpr int NL = 64 * CPR / kProThreads;
    static_assert(64 * CPR % kProThreads == 0, "other-half rows per thread");
    uint32_t mqb = 0u;
    {
        const int ro = half == 0 ? i0 + kAuxRows : i0 - kProQLo;   // the other half's rows
#pragma unroll
        for (int u = 0; u < NL; ++u) {
            const int row = ro + tid / CPR + u * RP;
            if (row >= 0 && row < T) {
                const uint4 v = *(const uint4 *)(q + head_off + (size_t)row * D + 8 * c8);
                mqb = absmax_bits(absmax_bits(absmax_bits(absmax_bits(mqb, v.x), v.y), v.z), v.w);
            }
        }
    }
    tc::cp_async_wait_all();
    __syncthreads();
    for (int lr = tid / CPR; lr < QR; lr += RP) {
        const uint4 v = *(const uint4 *)(qsm + lr * RS + 8 * c8);
        mqb = absmax_bits(absmax_bits(absmax_bits(absmax_bits(mqb, v.x), v.y), v.z), v.w);
    }
    const float mq = bits_to_absmax(mqb);
    __shared__ float red[8];
    int eq = range_exponent(block_max(mq, red));
    if (eq != 0 && tid == 0 && half == 0) atomicOr(&g_fused_error, kErrRange);   // see the fold
    if (eq < 0) eq = 0;
    if (tid == 0 && half == 0) qexp[(size_t)bh * nqb + qblk] = eq;
    const float qsc = ldexpf(1.f, -eq);       // exact: a power of two
    // (b) permuted query rows of the 128-row block jb0 = j0 - 64*half: atom a,
    //     row s <- q_{jb0-(c_q-1)+a+16s}; this CTA writes rows s in
    //     [4*half, 4*half+4), which lie in its copy [j0-7, j0+64) since
    //     c_q <= 8; 8 elements per thread
    {
        const int NA = q_atoms(c_q);
        __half *dst = qp + ((size_t)bh * (Tp / kBM) + qblk) * (size_t)NA * 8 * D;
        bool range_ok = true;
        for (int rowh = tid / CPR; rowh < NA * 4; rowh += RP) {
            const int a = rowh / 4, sr = rowh % 4;                // atom, row within this half
            const int row = 8 * a + 4 * half + sr;                // row of the block's atom layout
            const int rq = kProQLo - (c_q - 1) + a + 16 * sr;    // copy row of q_i
            const uint4 in = *(const uint4 *)(qsm + rq * RS + 8 * c8);
            const __nv_bfloat162 *bp = (const __nv_bfloat162 *)&in;
            uint4 outv;
            __half2 *hp = (__half2 *)&outv;
            if (eq == 0) {                        // the block fits fp16 as it is
#pragma unroll
                for (int u = 0; u < 4; ++u) hp[u] = __float22half2_rn(__bfloat1622float2(bp[u]));
            } else {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    float2 f = __bfloat1622float2(bp[u]);
                    f.x *= qsc;
                    f.y *= qsc;
                    range_ok &= fabsf(f.x) <= 65504.f && fabsf(f.y) <= 65504.f;
                    hp[u] = __floats2half2_rn(f.x, f.y);
                }
            }
            *(uint4 *)(dst + (size_t)row * D + 8 * c8) = outv;
        }
        if (!range_ok) atomicOr(&g_fused_error, kErrRange);
    }
    // (c) future logits F[r][delta] = scale * q_r . k_{r+delta} from the copies,
    //     on tensor cores (mma.sync m16n8k16, bf16 products summed in fp32): warp
    //     w takes q rows rr in [16w, 16w+16) against k rows kr in [16w, 16w+32),
    //     which hold every band entry delta = kr - rr + 1 in [1, 14] of its rows;
    //     each (rr, delta) lands in exactly one accumulator element.
    const int Dm = d_m(c_q, c_k);
    {
        const int wp = tid / 32, l = tid % 32;
        if (wp < QRP / 16) {
            const int m0 = 16 * wp;
            float acc[4][4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int x = 0; x < 4; ++x) acc[j][x] = 0.f;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t af[4];
                ldsm_x4(af, qsm + (m0 + (l & 15)) * RS + 16 * ks + 8 * (l >> 4));
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint32_t bf[2];
                    ldsm_x2(bf, ksm + (m0 + 8 * j + (l & 7)) * RS + 16 * ks + 8 * ((l >> 3) & 1));
                    mma_16816_bf16(acc[j], af, bf);
                }
            }
            const int gq = l >> 2, tq = l & 3;
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const int rr = m0 + gq + 8 * (x >> 1);
                    const int kr = m0 + 8 * j + 2 * tq + (x & 1);
                    const int dl = kr - rr + 1;
                    if (rr < QR && dl >= 1 && dl <= kCorrW - 2) {
                        const int r = j0 - kProQLo + rr;
                        fs[rr * kFs + dl - 1] =
                            (r >= 0 && dl <= Dm && r + dl < T) ? acc[j][x] * scale : 0.f;
                    }
                }
        }
    }
    __syncthreads();
    // (d) correction rows: thread = one row i (tid % 64) and the 4 entries
    //     e = 4g .. 4g+3, g = tid / 64 (the same in a whole warp):
    //     corr[i][e] = sum over taps (i', jj) of thp[i'][jj] F[i - i'][delta],
    //     delta = i' + RT - jj - e.  With the taps padded and centred at RT
    //     every delta is a compile-time constant, so only the terms with
    //     1 <= delta <= 14 are emitted (F is zero past D_m and before the
    //     sequence; padded taps are zero).  Under the exact mask the terms
    //     with delta <= i' are dropped.
    {
        const int ir = tid % kAuxRows, g = tid / kAuxRows;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        switch (g) {
            case 0: corr_terms<CK, 0, EXACT>(acc, fs + (ir + kProQLo) * kFs, kFs, thp, c_q); break;
            case 1: corr_terms<CK, 4, EXACT>(acc, fs + (ir + kProQLo) * kFs, kFs, thp, c_q); break;
            case 2: corr_terms<CK, 8, EXACT>(acc, fs + (ir + kProQLo) * kFs, kFs, thp, c_q); break;
            default: corr_terms<CK, 12, EXACT>(acc, fs + (ir + kProQLo) * kFs, kFs, thp, c_q); break;
        }
        *(float4 *)(corr + ((size_t)bh * Tp + j0 + ir) * kCorrW + 4 * g) =
            make_float4(acc[0], acc[1], acc[2], acc[3]);
    }
}

// Dynamic shared memory of the aux role: bf16 copies of 80 query rows and
// 96 key rows (71 and 84 used, the rest zero), each padded by 8 elements.
size_t prologue_smem_bytes(int D)
{
    const int QRP = (kProQLo + kAuxRows + 15) / 16 * 16;
    return (size_t)(QRP + QRP + 16) * (D + 8) * sizeof(__nv_bfloat16);
}

__device__ __forceinline__ void launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void wait_prerequisites()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// The whole prologue as one launch of 3 * nqb * BH CTAs in two roles: CTA
// 3u + 1 folds the keys of 128-key block u (u = b*H*nqb + ...), CTAs 3u and
// 3u + 2 build the permuted queries and correction rows of the two 64-row
// halves of the same 128-row block.  The fold is bound by FP32 issue and the
// rest by load latency, so interleaving them puts both kinds of CTA on every
// SM and each hides the other; it also keeps the q and k rows of a block in
// L2 for the three CTAs that read them.  The dependent main kernel may be
// scheduled as soon as every CTA of this grid has started.
template <int D, int CK, bool EXACT>
__global__ void __launch_bounds__(kProThreads, 3)
k_fold(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
       const float *__restrict__ w_kq, __half *__restrict__ kf, __half *__restrict__ qp,
       float *__restrict__ corr, int *__restrict__ sexp, int T, int Tp, int H, int nqb, int c_q,
       int c_k, float scale)
{
    launch_dependents();
    const int u = blockIdx.x / 3, role = blockIdx.x % 3;
    const int bh = u / nqb, blk = u % nqb;
    if (role == 1)
        fold_keys_block<D, CK>(blk, bh, k, w_kq, kf, sexp + (size_t)gridDim.x / 3, T, Tp, H, nqb,
                               c_q, c_k, scale);
    else
        fold_aux_block<D, CK, EXACT>(2 * blk + role / 2, bh, q, k, w_kq, qp, corr, sexp, T, Tp, H,
                                     nqb, c_q, c_k, scale);
}

// ------------------------------------------------------------ main kernel

// PAIR (d = 128): two CTAs (consecutive 128-row query blocks of one head)
// share every MMA as one M = 256 tcgen05 operation; each CTA then loads only
// half of every Kf tile (64 keys) and half of the V columns.  Without PAIR
// (d = 64) a CTA loads whole tiles.
//
// Ring slots are 32 KB.  A Kf slot holds two shifts i' (16 KB each: 64 keys
// x 128 d, or 128 keys x 64 d); a V slot holds the V tiles of kVHeads output
// heads, whose PV products then run as one MMA chain of N = kVHeads * d
// (in a pair each CTA holds one head's tile, or one half of the single
// head's columns).  The issuer meets its gate once per slot.
template <int D, int CH, bool PAIR>
struct FusedCfg {
    static_assert(PAIR == (D == 128), "pairs serve d = 128, single CTAs d = 64");
    static constexpr int kChunks = D / 64;                  // 64-element (128-B) column chunks
    static constexpr int kKfRows = PAIR ? kBN / 2 : kBN;    // keys of a Kf tile held by this CTA
    static constexpr int kShiftBytes = kKfRows * D * 2;     // one shift of one Kf tile
    static constexpr int kSlotBytes = 2 * kShiftBytes;
    static constexpr int kStages = 4;
    // output heads per work item: their U accumulators take at most 256 TMEM
    // columns; a larger group is split into kSplits items that repeat the
    // QK^T and softmax work for their share of the output heads
    static constexpr int kCHU = CH * D <= 256 ? CH : 256 / D;
    static constexpr int kSplits = CH / kCHU;
    static constexpr int kVHeads = kCHU < 2 ? kCHU : 2;     // output heads per V slot
    static constexpr int kVSlots = kCHU / kVHeads;          // V slots per key tile
    static constexpr int kVN = kVHeads * D;                 // N of one PV MMA chain
    static constexpr int kVBytes = kVHeads * 16384;         // bytes of a V slot this CTA loads
    static constexpr int kMaxAtoms = 23;                    // q_atoms(8)
    static constexpr int kQChunkBytes = kMaxAtoms * 1024;
    static constexpr int kOffRing = kChunks * kQChunkBytes;
    static constexpr int kOffScr = kOffRing + kStages * kSlotBytes;   // band-tile scratch rows
    static constexpr int kOffCorr = kOffScr + ((kBM * kScrStride * 4 + 1023) / 1024) * 1024;
    static constexpr int kOffBar = kOffCorr + kBM * kCorrStride * 4;
    static constexpr int kSmemBytes = kOffBar + 256 + 1024;  // + alignment slack
    static_assert(kShiftBytes == 16384 && kVN <= 256, "slot layout");
};

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Bounded wait: false when the budget ran out (the CTA's abort flag and the
// device error word are then set) or another role already aborted.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                         long long budget = kWaitBudget)
{
    if (tc::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (tc::mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > budget) {
            *abort_flag = 1;
            atomicOr(&g_fused_error, kErrTimeout);
            return false;
        }
    }
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b)
{
    __half2 v = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Bounded wait used by every role; in pair mode barriers that the other CTA
// arrives on are waited on with cluster-scope acquire.
template <bool PAIR>
__device__ __forceinline__ bool wait_role(uint64_t *bar, uint32_t parity, volatile int *abort_flag)
{
    if constexpr (!PAIR) {
        return wait_bar(bar, parity, abort_flag);
    } else {
        if (tc::mbar_try_wait_cluster(bar, parity)) return true;
        const long long t0 = clock64();
        while (true) {
            if (tc::mbar_try_wait_cluster(bar, parity)) return true;
            if (*abort_flag) return false;
            if (clock64() - t0 > kWaitBudget) {
                *abort_flag = 1;
                atomicOr(&g_fused_error, kErrTimeout);
                return false;
            }
        }
    }
}

// Arrival on a barrier of the MMA-issuing CTA (rank 0 of a pair, or self).
// Its only use publishes P~ (and a rescaled U): TMEM data whose stores the
// arriving warp has waited for and fenced before the arrival, and which the
// issuer reads only through MMAs it issues after an acquire wait on the
// barrier and tcgen05.fence::after_thread_sync.  No generic-memory data rides
// on it, so the pair form is a relaxed arrival: a release at cluster scope
// held each softmax warp about 1500 cycles per key tile.
template <bool PAIR>
__device__ __forceinline__ void arrive_leader(uint64_t *bar)
{
    if constexpr (PAIR) tc::mbar_arrive_cluster_relaxed(tc::mapa_shared(tc::smem_u32(bar), 0));
    else tc::mbar_arrive(bar);
}

// Work items of the persistent main kernel: (b, h, query block) without
// pairs, (b, h, pair of blocks) with them.  The list is ordered by decreasing
// length (key tiles), and cluster cl takes one item per round, snaking across
// the clusters (left to right in even rounds, right to left in odd ones), so
// every role derives the same sequence with no communication.
struct WorkItem {
    int bh, b, g, hl, hh0, qb, i0, ntiles;
};

template <bool PAIR>
__device__ __forceinline__ bool work_item(int k, int cl, int ncl, int BH, int H, int CH,
                                          int chu, int nqb, uint32_t rank, WorkItem &it)
{
    const int per_head = PAIR ? nqb / 2 : nqb;
    const int splits = CH / chu;
    const int pos = k * ncl + ((k & 1) ? ncl - 1 - cl : cl);
    if (pos >= per_head * BH * splits) return false;
    const int cls = pos / (BH * splits), rem = pos % (BH * splits);
    const int bhx = rem / splits;
    it.hh0 = (rem % splits) * chu;            // first output head of the item
    const int hs = bhx % H;
    it.bh = bhx;
    it.b = bhx / H;
    it.g = hs / CH;
    it.hl = hs % CH;
    if (PAIR) {
        const int pair = per_head - 1 - cls;
        it.qb = 2 * pair + (int)rank;
        it.ntiles = 2 * pair + 2;     // both CTAs run to the diagonal of block 2p+1
    } else {
        it.qb = nqb - 1 - cls;
        it.ntiles = it.qb + 1;
    }
    it.i0 = it.qb * kBM;
    return true;
}

// Block 224 threads = warp 0 TMA producer,
// warp 1 MMA issuer (and TMEM owner), warps 2..5 softmax / epilogue (one TMEM
// lane, i.e. one query row, per thread), warp 6 gate of the issuer.  TMEM columns: S double buffer at
// 0 and 128, U^{h,h'} for the c_h output heads from 256.
// PAIR (d = 128): clusters of two CTAs own query blocks 2p and 2p+1 of one
// head; rank 0 issues the M = 256 MMAs for both and every completion is
// multicast to both CTAs' barriers.
template <int D, int CH, bool PAIR>
__global__ void __launch_bounds__(224, 1)
k_mta_fused(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
            const __grid_constant__ CUtensorMap mapV, const float *__restrict__ corr,
            const int *__restrict__ sexp, const float *__restrict__ w_head,
            __half *__restrict__ part, int T, int Tp, int H, int c_q, int nqb, int nbh)
{
    using C = FusedCfg<D, CH, PAIR>;
    static_assert(C::kStages <= kGateQ - kGateStage0, "one gate barrier id per ring slot");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *sQ = base;
    uint8_t *ring = base + C::kOffRing;
    float *sScr = (float *)(base + C::kOffScr);
    float *sCorr = (float *)(base + C::kOffCorr);
    uint64_t *bar_q = (uint64_t *)(base + C::kOffBar);
    uint64_t *full = bar_q + 1;
    uint64_t *empty = full + C::kStages;
    uint64_t *s_full = empty + C::kStages;
    uint64_t *p_full = s_full + 2;
    uint64_t *pv_done = p_full + 1;
    uint64_t *mma_drain = pv_done + 1;

    uint64_t *q_free = mma_drain + 1;
    uint32_t *tmem_slot = (uint32_t *)(q_free + 1);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);

    // Persistent grid: cluster cl of ncl walks its work items (work_item);
    // every role keeps its ring slot, barrier phases and the global key-tile
    // counter gt running across items.
    const uint32_t rank = PAIR ? tc::cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    const int ncl = PAIR ? (int)gridDim.x / 2 : (int)gridDim.x;
    const int cl = PAIR ? (int)blockIdx.x / 2 : (int)blockIdx.x;
    const int BH = nbh;
    const int NA = q_atoms(c_q);
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int consumers = PAIR ? 8 : 4;   // softmax warps that publish P~
    const int kf_slots = (c_q + 1) / 2;
    auto item = [&](int k, WorkItem &it) {
        return work_item<PAIR>(k, cl, ncl, BH, H, CH, C::kCHU, nqb, rank, it);
    };

    if (threadIdx.x == 0) {
        tc::mbar_init(bar_q, 1);
        for (int s = 0; s < C::kStages; ++s) { tc::mbar_init(&full[s], 1); tc::mbar_init(&empty[s], 1); }
        tc::mbar_init(&s_full[0], 1); tc::mbar_init(&s_full[1], 1);
        tc::mbar_init(p_full, consumers);
        tc::mbar_init(pv_done, 1);
        tc::mbar_init(mma_drain, 1);
        tc::mbar_init(q_free, 1);
        *abort_flag = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) {
        if constexpr (PAIR) { tc::tmem_alloc_pair(tmem_slot, 512); tc::tmem_relinquish_pair(); }
        else { tc::tmem_alloc(tmem_slot, 512); tc::tmem_relinquish(); }
    }
    tc::tc_fence_before();
    __syncthreads();
    if constexpr (PAIR) tc::cluster_sync();   // the peer's barriers exist before any remote use
    tc::tc_fence_after();
    const uint32_t tm = *tmem_slot;
    // everything above overlaps the prologue's tail; its outputs (Kf, the
    // permuted queries, the correction rows) are read only after this
    wait_prerequisites();

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer
            tc::prefetch_tmap(&mapQ); tc::prefetch_tmap(&mapK); tc::prefetch_tmap(&mapV);
            const uint32_t q_bytes = C::kChunks * NA * 8 * 128;
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_phase[C::kStages];
            bool issued[C::kStages];
            for (int s = 0; s < C::kStages; ++s) issued[s] = false;
            bool ok = true;
            int q_loads = 0;
            // Claims the next ring slot and counts `bytes` (this CTA's part) on
            // its full barrier; the leader of a pair expects both CTAs' parts.
            auto claim = [&](uint32_t bytes) -> uint8_t * {
                if (!wait_role<PAIR>(&empty[stage], phase ^ 1, abort_flag)) return nullptr;
                if (leader) tc::mbar_arrive_expect_tx(&full[stage], PAIR ? 2 * bytes : bytes);
                return ring + stage * C::kSlotBytes;
            };
            auto advance = [&]() {
                issued[stage] = true;
                issued_phase[stage] = phase;
                if (++stage == C::kStages) { stage = 0; phase ^= 1; }
            };
            auto tile_load = [&](uint8_t *dst, const CUtensorMap *map, int x, int y, int z) {
                if constexpr (PAIR)
                    tc::tma_load_3d_pair(dst, map, tc::mapa_shared(tc::smem_u32(&full[stage]), 0), x, y, z);
                else
                    tc::tma_load_3d(dst, map, &full[stage], x, y, z);
            };
            // the permuted Q block of an item, once the previous item's last
            // QK MMAs have finished reading the buffer
            auto load_q = [&](const WorkItem &it) -> bool {
                if (q_loads > 0 && !wait_role<PAIR>(q_free, (q_loads - 1) & 1, abort_flag)) return false;
                if (leader) tc::mbar_arrive_expect_tx(bar_q, PAIR ? 2 * q_bytes : q_bytes);
                const uint32_t bq = tc::mapa_shared(tc::smem_u32(bar_q), 0);
                for (int c = 0; c < C::kChunks; ++c) {
                    if constexpr (PAIR) tc::tma_load_3d_pair(sQ + c * C::kQChunkBytes, &mapQ, bq, 64 * c, it.qb * NA * 8, it.bh);
                    else tc::tma_load_3d(sQ + c * C::kQChunkBytes, &mapQ, bar_q, 64 * c, it.qb * NA * 8, it.bh);
                }
                ++q_loads;
                return true;
            };
            // Kf slot m of key tile t: shifts 2m and 2m+1 (when below c_q)
            auto load_kf = [&](const WorkItem &it, int t, int m) -> bool {
                const int n = (2 * m + 1 < c_q) ? 2 : 1;
                uint8_t *dst = claim(n * C::kShiftBytes);
                if (dst == nullptr) return false;
                for (int h = 0; h < n; ++h)
                    for (int c = 0; c < C::kChunks; ++c)
                        tile_load(dst + h * C::kShiftBytes + c * (C::kKfRows * 128), &mapK, 64 * c,
                                  t * kBN + (PAIR ? (int)rank * C::kKfRows : 0), it.bh * c_q + 2 * m + h);
                advance();
                return true;
            };
            // V slot vs of key tile u: heads vs*kVHeads ...; in a pair with two
            // heads CTA r loads head r whole, with one head it loads column half r
            auto load_v = [&](const WorkItem &it, int u, int vs) -> bool {
                uint8_t *dst = claim(C::kVBytes);
                if (dst == nullptr) return false;
                const int z0 = it.b * H + it.g * CH + it.hh0 + vs * C::kVHeads;
                if constexpr (PAIR) {
                    if (C::kVHeads == 2) {
                        for (int c = 0; c < C::kChunks; ++c)
                            tile_load(dst + c * 16384, &mapV, 64 * c, u * kBN, z0 + (int)rank);
                    } else {
                        tile_load(dst, &mapV, 64 * (int)rank, u * kBN, z0);
                    }
                } else {
                    for (int j = 0; j < C::kVHeads; ++j) tile_load(dst + j * 16384, &mapV, 0, u * kBN, z0 + j);
                }
                advance();
                return true;
            };
            // slot order = the issuer's: per item, Kf(t) then V(t-1) for each
            // tile, and the item's last V right after its last Kf
            WorkItem it, nx;
            bool have = item(0, it);
            for (int k = 0; have && ok; ++k) {
                const bool have_next = item(k + 1, nx);
                for (int t = 0; t < it.ntiles && ok; ++t) {
                    for (int m = 0; m < kf_slots && ok; ++m) ok = load_kf(it, t, m);
                    if (ok && t == 0) ok = load_q(it);
                    // the next item's Q block into L2 while this item's last
                    // tile runs.  (Prefetching key tiles ahead as well was
                    // measured slower: the prefetches compete with the ring's
                    // own loads.)
                    if (have_next && t == it.ntiles - 1)
                        for (int c = 0; c < C::kChunks; ++c)
                            tc::tma_prefetch_3d(&mapQ, 64 * c, nx.qb * NA * 8, nx.bh);
                    for (int vs = 0; vs < C::kVSlots && ok && t > 0; ++vs) ok = load_v(it, t - 1, vs);
                }
                for (int vs = 0; vs < C::kVSlots && ok; ++vs) ok = load_v(it, it.ntiles - 1, vs);
                it = nx;
                have = have_next;
            }
            // copies this thread started land before the CTA may exit; in a pair
            // their completion is counted in the leader, so the peer waits a while
            if (leader) {
                if (q_loads > 0) tc::mbar_wait(bar_q, (q_loads - 1) & 1, kWaitBudget);
                for (int s = 0; s < C::kStages; ++s)
                    if (issued[s]) tc::mbar_wait(&full[s], issued_phase[s], kWaitBudget);
            } else if (!ok) {
                const long long t0 = clock64();
                while (clock64() - t0 < (1ll << 22)) { }
            }
        }
    } else if (warp == 1) {
        if (leader) {
            // ---------------- MMA issuer: lane 0 issues, the whole warp meets
            // the gate warp at one named barrier per step, so no shared-memory
            // access sits in the issue stream.
            const bool issuer = lane == 0;
            // Descriptors are built once; the start-address field holds
            // address >> 4, so every tile, stage and K step below is one add.
            constexpr int M = PAIR ? 2 * kBM : kBM;
            const uint32_t idq = tc::idesc_f16(M, kBN, false, false);
            const uint32_t idv = tc::idesc_bf16(M, C::kVN, false, true);
            const uint64_t dq0 = tc::sdesc_sw128(tc::smem_u32(sQ), 16, 1024);
            const uint64_t dk0 = tc::sdesc_sw128(tc::smem_u32(ring), 16, 1024);
            // V is MN-major: 64-column chunks of one slot lie 16 KB apart
            const uint64_t dv0 = tc::sdesc_sw128(tc::smem_u32(ring), 16384, 1024);
            auto mma = [&](uint32_t d, uint64_t ad, uint64_t bd, uint32_t id, uint32_t acc) {
                if constexpr (PAIR) tc::mma_pair(d, ad, bd, id, acc);
                else tc::mma_bf16(d, ad, bd, id, acc);
            };
            auto mma_t = [&](uint32_t d, uint32_t at, uint64_t bd, uint32_t id, uint32_t acc) {
                if constexpr (PAIR) tc::mma_pair_ts(d, at, bd, id, acc);
                else tc::mma_ts(d, at, bd, id, acc);
            };
            auto commit = [&](uint64_t *bar) {
                if constexpr (PAIR) tc::mma_commit_pair_multicast(bar, 0x3);
                else tc::mma_commit(bar);
            };
            auto gate = [&](int id) {
                __syncwarp();
                tc::named_bar_sync(id, 64);
            };
            int stage = 0;
            // The TMA data behind a full barrier needs no tcgen05 fence; P~ (in
            // TMEM over the first half of its S buffer) and the rescaled U,
            // which the gate also waited for before the first V slot, do.
            // S(g+2) overwrites the buffer only after PV(g), which reads P~(g),
            // has been issued: the pipe executes in issue order.  PV of an
            // item's first tile overwrites U (the softmax warps read the
            // previous item's U before they publish that tile's P~).
            auto issue_pv = [&](int gprev, int tprev) {
                for (int vs = 0; vs < C::kVSlots; ++vs) {
                    gate(kGateStage0 + stage);
                    if (vs == 0) tc::tc_fence_after();
                    if (issuer) {
                        const uint64_t bv = dv0 + (uint64_t)((stage * C::kSlotBytes) >> 4);
#pragma unroll
                        for (int kk = 0; kk < kBN / 16; ++kk)
                            mma_t(tm + 256 + vs * C::kVN, tm + (gprev & 1) * kBN + kk * 8,
                                  bv + (uint64_t)((kk * 2048) >> 4), idv, (tprev > 0 || kk > 0) ? 1u : 0u);
                        commit(&empty[stage]);
                    }
                    if (++stage == C::kStages) stage = 0;
                }
                if (issuer) commit(pv_done);
            };
            int gt = 0;
            WorkItem it;
            for (int k = 0; item(k, it); ++k) {
                gate(kGateQ);                  // this item's Q block has landed
                for (int t = 0; t < it.ntiles; ++t, ++gt) {
                    const int sb = gt & 1;
                    for (int m = 0; m < kf_slots; ++m) {
                        gate(kGateStage0 + stage);
                        if (issuer) {
                            const uint64_t bs = dk0 + (uint64_t)((stage * C::kSlotBytes) >> 4);
                            for (int h = 0; h < 2; ++h) {
                                const int ip = 2 * m + h;
                                if (ip >= c_q) break;
                                const uint64_t aq = dq0 + (uint64_t)(((c_q - 1 - ip) * 1024) >> 4);
                                const uint64_t bk = bs + (uint64_t)((h * C::kShiftBytes) >> 4);
#pragma unroll
                                for (int c = 0; c < C::kChunks; ++c)
#pragma unroll
                                    for (int kk = 0; kk < 4; ++kk)
                                        mma(tm + sb * kBN, aq + (uint64_t)((c * C::kQChunkBytes + kk * 32) >> 4),
                                            bk + (uint64_t)((c * (C::kKfRows * 128) + kk * 32) >> 4), idq,
                                            (ip | c | kk) ? 1u : 0u);
                            }
                            commit(&empty[stage]);
                        }
                        if (++stage == C::kStages) stage = 0;
                    }
                    if (issuer) {
                        commit(&s_full[sb]);
                        if (t == it.ntiles - 1) commit(q_free);   // the Q block may be replaced
                    }
                    if (t > 0) issue_pv(gt - 1, t - 1);
                }
                // the item's last PV before the next item's first QK: its
                // partial outputs can be written while that QK runs
                issue_pv(gt - 1, it.ntiles - 1);
            }
            // all MMAs this warp issued complete before TMEM is released
            if (issuer) {
                if constexpr (PAIR) tc::mma_commit_pair_multicast(mma_drain, 0x1);
                else tc::mma_commit(mma_drain);
                tc::mbar_wait(mma_drain, 0, kWaitBudget);
            }
        }
    } else if (warp == 6) {
        if (leader) {
            // ---------------- gate: waits, in the issuer's order, for each
            // barrier the next MMA step depends on and arrives (without
            // blocking) at that ring slot's named barrier, so it runs ahead of
            // the issuer.  A slot's barrier never receives a second arrival
            // before the issuer has consumed the first: the slot is refilled
            // only after the issuer's commit for its previous use.  The first
            // V slot of PV(u) also waits for P~(u) (p_full).  After a timeout
            // or abort the gate stops waiting on data but still arrives at
            // every meeting, each time after the issuer's commit for the
            // slot's previous use, so the issuer runs to its end and drains.
            bool ok = true;
            int stage = 0;
            uint32_t phase = 0;
            auto meet = [&](bool with_p, int u) {
                int r = 1;
                if (lane == 0) {
                    if (ok && with_p) r = wait_role<PAIR>(p_full, u & 1, abort_flag) ? 1 : 0;
                    if (ok && r) r = wait_role<PAIR>(&full[stage], phase, abort_flag) ? 1 : 0;
                    if (!ok || !r) tc::mbar_wait(&empty[stage], phase ^ 1, kWaitBudget);
                }
                ok = ok && __shfl_sync(0xffffffffu, r, 0) != 0;
                __syncwarp();
                tc::named_bar_arrive(kGateStage0 + stage, 64);
                if (++stage == C::kStages) { stage = 0; phase ^= 1; }
            };
            // Q block of item k; after an abort, only once the issuer's commit
            // after the previous item's last QK shows it consumed the last meeting
            auto meet_q = [&](int k) {
                int r = 1;
                if (lane == 0) {
                    if (ok) r = wait_role<PAIR>(bar_q, k & 1, abort_flag) ? 1 : 0;
                    if ((!ok || !r) && k > 0) tc::mbar_wait(q_free, (k - 1) & 1, kWaitBudget);
                }
                ok = ok && __shfl_sync(0xffffffffu, r, 0) != 0;
                __syncwarp();
                tc::named_bar_arrive(kGateQ, 64);
            };
            int gt = 0;
            WorkItem it;
            for (int k = 0; item(k, it); ++k) {
                meet_q(k);
                for (int t = 0; t < it.ntiles; ++t, ++gt) {
                    for (int m = 0; m < kf_slots; ++m) meet(false, 0);
                    for (int vs = 0; vs < C::kVSlots && t > 0; ++vs) meet(vs == 0, gt - 1);
                }
                for (int vs = 0; vs < C::kVSlots; ++vs) meet(vs == 0, gt - 1);
            }
        }
    } else {
        // ---------------- softmax and epilogue (warps 2..5): thread = TMEM lane = one query row
        const int q4 = warp & 3;                       // lane quarter this warp may access
        const int r = q4 * 32 + lane;
        const uint32_t lane_base = tm + ((uint32_t)(q4 * 32) << 16);
        float *crow = sCorr + r * kCorrStride;
        float *scr = sScr + r * kScrStride;   // this thread's scratch row (band tiles, epilogue)
        bool ok = true;
        int gt = 0;
        WorkItem it, nx;
        // this row's correction entries of an item (read an item ahead, so
        // that the load overlaps the previous item's epilogue)
        float4 cnext[kCorrW / 4];
        auto fetch_corr = [&](const WorkItem &w) {
            const int ir = w.i0 + 16 * (r & 7) + (r >> 3);
            const float4 *src = (const float4 *)(corr + ((size_t)w.bh * Tp + ir) * kCorrW);
#pragma unroll
            for (int u = 0; u < kCorrW / 4; ++u) cnext[u] = src[u];
        };
        bool have = item(0, it);
        if (have) fetch_corr(it);
        for (int k = 0; ok && have; ++k) {
            const int qb = it.qb, i0 = it.i0, b = it.b, g = it.g, hl = it.hl;
#pragma unroll
            for (int u = 0; u < kCorrW / 4; ++u) {
                crow[4 * u] = cnext[u].x; crow[4 * u + 1] = cnext[u].y;
                crow[4 * u + 2] = cnext[u].z; crow[4 * u + 3] = cnext[u].w;
            }
            const bool have_next = item(k + 1, nx);
            float m_run = -INFINITY, l = 0.f;
            // range exponents of this CTA's query block and of each key tile
            // (zero unless the prologue scaled a block's fp16 operands down)
            const int eq = sexp[(size_t)it.bh * nqb + qb];
            const int *ekp = sexp + (size_t)BH * nqb + (size_t)it.bh * nqb;
            for (int t = 0; t < it.ntiles; ++t, ++gt) {
                const int sb = gt & 1;
                const int escale = eq + ekp[t];
                ok = __all_sync(0xffffffffu, wait_role<PAIR>(&s_full[sb], (gt >> 1) & 1, abort_flag));
                if (!ok) break;
                tc::tc_fence_after();
                // The first block of a pair runs one tile past its diagonal: every
                // key there is in the future, so P~ is zero and the row state stays.
                const bool live = t <= qb;
                uint32_t pk[kBN / 2];
                float lp[8];
                bool need = false;
                float m_new = m_run, alpha = 1.f;
#pragma unroll
                for (int x = 0; x < 8; ++x) lp[x] = 0.f;
                if (live) {
                float s[kBN];
#pragma unroll
                for (int j = 0; j < kBN / 32; ++j) tc::tmem_ld32f(lane_base + sb * kBN + 32 * j, s + 32 * j);
                tc::tmem_ld_wait();
                if (escale != 0) {      // undo the blocks' operand scaling (exact)
                    const float f = ldexpf(1.f, escale);
#pragma unroll
                    for (int c = 0; c < kBN; ++c) s[c] *= f;
                }
                // Band tiles (this block's diagonal tile and the one before it):
                // for key j0 + c the diagonal offset is e = i_row - j0 - c; keys
                // with e < 0 are in the future (-inf), and the Mask_0 correction
                // corr[i][e] (nonzero for e < D_m < kCorrW = 16) is subtracted.
                // With the permuted row order i_row - i0 = 16 a + beta (a = lane & 7,
                // beta = 4 q4 + lane / 8) and c = 16 a' + gamma, the diagonal tile
                // has e = 16 (a - a') + beta - gamma: e lies in [0, 16) only for
                // a' = a, gamma <= beta, or a' = a - 1, gamma > beta, and then
                // corr[e] = corr[(beta - gamma) mod 16].  So 16 table reads per
                // row serve the whole tile and the rest is register selects.  The
                // tile before the diagonal has e >= 1, and e < 16 only in the rows
                // with a = 0, at columns c = 112 + gamma with gamma > beta.
                if (t >= qb - 1) {
                    const int a = lane & 7, beta = 4 * q4 + (lane >> 3);
                    float w[kCorrW];
#pragma unroll
                    for (int gm = 0; gm < kCorrW; ++gm) w[gm] = crow[(beta - gm) & (kCorrW - 1)];
                    if (t == qb) {
#pragma unroll
                        for (int a2 = 0; a2 < kBN / 16; ++a2) {
                            const bool same = a2 == a, prev = a2 == a - 1, later = a2 > a;
#pragma unroll
                            for (int gm = 0; gm < 16; ++gm) {
                                const int c = 16 * a2 + gm;
                                const bool band = (gm <= beta) ? same : prev;
                                const bool future = later || (same && gm > beta);
                                const float v = s[c] - (band ? w[gm] : 0.f);
                                s[c] = future ? -INFINITY : v;
                            }
                        }
                    } else if (a == 0) {
#pragma unroll
                        for (int gm = 0; gm < 16; ++gm)
                            if (gm > beta) s[kBN - 16 + gm] -= w[gm];
                    }
                }
                // row max as 8 independent partial maxima
                float mp[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) mp[x] = s[x];
#pragma unroll
                for (int c = 8; c < kBN; ++c) mp[c & 7] = fmaxf(mp[c & 7], s[c]);
                const float mt = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                                       fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
                // the running max moves only when it grows by more than 2^8 in scale
                need = mt > m_run + 8.f;
                m_new = need ? mt : m_run;
                alpha = ex2(m_run - m_new);
                // P~ = exp2(S - m), packed to bf16 pairs; each half goes to TMEM
                // (over the first kBN/2 columns of the S buffer, where PV(t) reads
                // it as the A operand) as soon as it is ready, so the first store
                // overlaps the second half's exponentials
#pragma unroll
                for (int c = 0; c < kBN / 2; c += 2) {
                    const float p0 = ex2(s[c] - m_new), p1 = ex2(s[c + 1] - m_new);
                    lp[(c >> 1) & 7] += p0 + p1;
                    pk[c >> 1] = pack_bf16(p0, p1);
                }
                tc::tmem_st32(lane_base + sb * kBN, *reinterpret_cast<const uint32_t(*)[32]>(pk));
#pragma unroll
                for (int c = kBN / 2; c < kBN; c += 2) {
                    const float p0 = ex2(s[c] - m_new), p1 = ex2(s[c + 1] - m_new);
                    lp[(c >> 1) & 7] += p0 + p1;
                    pk[c >> 1] = pack_bf16(p0, p1);
                }
                tc::tmem_st32(lane_base + sb * kBN + 32, *reinterpret_cast<const uint32_t(*)[32]>(pk + 32));
                } else {
#pragma unroll
                    for (int x = 0; x < kBN / 2; ++x) pk[x] = 0u;
                    tc::tmem_st32(lane_base + sb * kBN, *reinterpret_cast<const uint32_t(*)[32]>(pk));
                    tc::tmem_st32(lane_base + sb * kBN + 32, *reinterpret_cast<const uint32_t(*)[32]>(pk + 32));
                }
                // Every warp waits for PV(t-1) to complete before it publishes
                // P~(t).  p_full counts arrivals from all softmax warps (of both
                // CTAs in a pair); without this wait a warp that ran a tile ahead
                // could complete phase t for a warp still working on tile t.  The
                // wait also orders the (rare) rescale of U after PV(t-1) added
                // into it.
                if (gt > 0) {
                    ok = __all_sync(0xffffffffu, wait_role<PAIR>(pv_done, (gt - 1) & 1, abort_flag));
                    if (!ok) break;
                    tc::tc_fence_after();
                }
                if (t > 0 && __any_sync(0xffffffffu, need)) {
                    const float f = need ? alpha : 1.f;
#pragma unroll
                    for (int hh = 0; hh < C::kCHU; ++hh)
#pragma unroll
                        for (int j = 0; j < D / 32; ++j) {
                            uint32_t u[32];
                            const uint32_t a = lane_base + 256 + hh * D + 32 * j;
                            tc::tmem_ld32(a, u);
                            tc::tmem_ld_wait();
#pragma unroll
                            for (int x = 0; x < 32; ++x) u[x] = __float_as_uint(__uint_as_float(u[x]) * f);
                            tc::tmem_st32(a, u);
                        }
                }
                l = l * alpha + (((lp[0] + lp[1]) + (lp[2] + lp[3])) + ((lp[4] + lp[5]) + (lp[6] + lp[7])));
                m_run = m_new;
                // P~(t) is in TMEM once the stores issued above have completed
                tc::tmem_st_wait();
                tc::tc_fence_before();
                __syncwarp();
                if (lane == 0) arrive_leader<PAIR>(p_full);
            }
            if (!ok) break;
            if (have_next) fetch_corr(nx);
            const int hh0 = it.hh0;
            float coef[C::kCHU];
#pragma unroll
            for (int hh = 0; hh < C::kCHU; ++hh) coef[hh] = w_head[((size_t)g * CH + hh0 + hh) * CH + hl];
            // the item's last PV has completed: write its partial outputs
            ok = __all_sync(0xffffffffu, wait_role<PAIR>(pv_done, (gt - 1) & 1, abort_flag));
            if (ok) {
                // (w_head / l) U in fp16, one head's d columns loaded from TMEM at
                // once, written 64 columns (128 B) at a time: each thread puts its
                // row's 64 values into its scratch row, then every 16-B store of
                // the warp covers, with 8 lanes, the 128-B segment of one of 4 rows
                tc::tc_fence_after();
                const float inv_l = 1.f / l;
                const size_t row_stride = (size_t)H * CH * D;
#pragma unroll 1
                for (int hh = 0; hh < C::kCHU; ++hh) {
                    const float cf = coef[hh] * inv_l;
                    __half *dst = part + (size_t)b * T * row_stride + (size_t)(g * CH + hh0 + hh) * (CH * D) + hl * D;
                    uint32_t u[D];
#pragma unroll
                    for (int j = 0; j < D / 32; ++j)
                        tc::tmem_ld32(lane_base + 256 + hh * D + 32 * j, *reinterpret_cast<uint32_t(*)[32]>(u + 32 * j));
                    tc::tmem_ld_wait();
                    uint32_t *srow = reinterpret_cast<uint32_t *>(scr);
#pragma unroll
                    for (int j = 0; j < D / 64; ++j) {
                        __syncwarp();
#pragma unroll
                        for (int x = 0; x < 32; x += 4) {
                            uint4 w4;
                            const int c = 64 * j + 2 * x;
                            w4.x = pack_h2(__uint_as_float(u[c]) * cf, __uint_as_float(u[c + 1]) * cf);
                            w4.y = pack_h2(__uint_as_float(u[c + 2]) * cf, __uint_as_float(u[c + 3]) * cf);
                            w4.z = pack_h2(__uint_as_float(u[c + 4]) * cf, __uint_as_float(u[c + 5]) * cf);
                            w4.w = pack_h2(__uint_as_float(u[c + 6]) * cf, __uint_as_float(u[c + 7]) * cf);
                            *(uint4 *)(srow + x) = w4;
                        }
                        __syncwarp();
#pragma unroll
                        for (int rho = 0; rho < 8; ++rho) {
                            const int rr = q4 * 32 + 4 * rho + (lane >> 3);
                            const int ir = i0 + 16 * (rr & 7) + (rr >> 3);
                            const uint4 v = *(const uint4 *)(sScr + rr * kScrStride + 4 * (lane & 7));
                            if (ir < T) *(uint4 *)(dst + (size_t)ir * row_stride + 64 * j + 8 * (lane & 7)) = v;
                        }
                    }
                }
            }
            it = nx;
            have = have_next;
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    // this CTA's work is done: the GroupNorm kernel may be scheduled
    launch_dependents();
    // in a pair, the leader's MMAs touch both CTAs' TMEM and shared memory
    if constexpr (PAIR) tc::cluster_sync();
    if (warp == 1) {
        tc::tc_fence_after();
        if constexpr (PAIR) tc::tmem_dealloc_pair(tm, 512);
        else tc::tmem_dealloc(tm, 512);
    }
}

// One thread waits, with the fused kernels' bounded wait, on a barrier that
// expects an arrival nobody makes; the wait gives up after `budget` cycles.
__global__ void k_selftest_wait_timeout(long long budget)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    tc::mbar_init(&bar, 1);
    abort_flag = 0;
    tc::fence_barrier_init();
    wait_bar(&bar, 0, &abort_flag, budget);
}

// ------------------------------------------------------------ mix + GroupNorm

// Thread = 8 consecutive channels e0..e0+7 of one (b, t, h); the d/8 threads
// of a head are consecutive lanes of one warp (16 at d = 128, 8 at d = 64).
// O^h = sum_{h'} part[b][t][h][h'] (fp16 partials, one 16-byte load per
// source head, summed in fp32), then GroupNorm over the head's d values
// (mean and biased variance by shuffles within the lane group), affine, and
// the head's scale: the depth scale, or sigmoid(g_h) ("Group Normalization
// with Sigmoid Gating").  One 16-byte bf16 store per thread.
constexpr int kMixThreads = 256;

template <int D, int CH>
__global__ void __launch_bounds__(kMixThreads)
k_mix_groupnorm(const __half *__restrict__ part, const float *__restrict__ gn_weight,
                const float *__restrict__ gn_bias, float depth_scale,
                const float *__restrict__ gate, float eps, __nv_bfloat16 *__restrict__ out,
                int T, int H, long long units)
{
    constexpr int G = D / 8;                   // threads per (b, t, h)
    const long long u0 = (long long)blockIdx.x * (kMixThreads / G) + threadIdx.x / G;
    const bool live = u0 < units;              // the grid's last warp may be partly past the end:
    const long long u = live ? u0 : units - 1; // its lanes recompute a valid unit, store nothing
    const int e0 = 8 * (threadIdx.x % G);
    wait_prerequisites();                      // the partial outputs are complete
    const int h = (int)(u % H);
    const long long bt = u / H;                // b * T + t
    const uint4 *src = (const uint4 *)(part + (bt * H + h) * (long long)(CH * D) + e0);
    uint4 raw[CH];
#pragma unroll
    for (int hs = 0; hs < CH; ++hs) raw[hs] = src[hs * (D / 8)];
    float o[8];
#pragma unroll
    for (int x = 0; x < 8; ++x) o[x] = 0.f;
#pragma unroll
    for (int hs = 0; hs < CH; ++hs) {
        const __half2 *hp = (const __half2 *)&raw[hs];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const float2 f = __half22float2(hp[x]);
            o[2 * x] += f.x;
            o[2 * x + 1] += f.y;
        }
    }
    float sum = 0.f;
#pragma unroll
    for (int x = 0; x < 8; ++x) sum += o[x];
#pragma unroll
    for (int m = G / 2; m > 0; m >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, m);
    const float mean = sum / D;
    float sq = 0.f;
#pragma unroll
    for (int x = 0; x < 8; ++x) sq += (o[x] - mean) * (o[x] - mean);
#pragma unroll
    for (int m = G / 2; m > 0; m >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, m);
    const float inv = 1.f / sqrtf(sq / D + eps);
    // the head's output scale: sigmoid(g_h), or the depth scale
    const float scale = gate ? 1.f / (1.f + expf(-gate[h])) : depth_scale;
    const float4 *gw = (const float4 *)(gn_weight + h * D + e0);
    const float4 *gb = (const float4 *)(gn_bias + h * D + e0);
    const float4 w0 = gw[0], w1 = gw[1], b0 = gb[0], b1 = gb[1];
    const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
    uint4 res;
    uint32_t *rp = (uint32_t *)&res;
    bool finite = true;
#pragma unroll
    for (int x = 0; x < 4; ++x) {
        const float y0 = scale * ((o[2 * x] - mean) * inv * wv[2 * x] + bv[2 * x]);
        const float y1 = scale * ((o[2 * x + 1] - mean) * inv * wv[2 * x + 1] + bv[2 * x + 1]);
        finite &= fabsf(y0) <= 3.0e38f && fabsf(y1) <= 3.0e38f;   // false for NaN too
        rp[x] = pack_bf16(y0, y1);
    }
    // an output that is not finite can only come from a non-finite q, k or v
    // (or one the fp16 operands could not hold): report it
    if (__any_sync(0xffffffffu, live && !finite) && threadIdx.x % 32 == 0)
        atomicOr(&g_fused_error, kErrRange);
    if (live) *(uint4 *)(out + bt * ((long long)H * D) + (long long)h * D + e0) = res;
}

// ------------------------------------------------------------ host side

struct FusedLayout {
    int Tp, nqb, NA;
    size_t off_kf, off_qp, off_corr, off_part, off_exp, total;
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

FusedLayout fused_layout(const mta_shape &s)
{
    FusedLayout L;
    L.Tp = (s.T + 2 * kBM - 1) / (2 * kBM) * (2 * kBM);   // an even number of query blocks
    L.nqb = L.Tp / kBM;
    L.NA = q_atoms(s.c_q);
    const size_t BH = (size_t)s.B * s.H;
    size_t off = 0;
    L.off_kf = off;   off += align256(BH * s.c_q * L.Tp * s.d * 2);
    L.off_qp = off;   off += align256(BH * L.nqb * L.NA * 8 * s.d * 2);
    L.off_corr = off; off += align256(BH * L.Tp * kCorrW * 4);
    L.off_part = off; off += align256((size_t)s.B * s.T * s.H * s.c_h * s.d * 2);
    L.off_exp = off;  off += align256(2 * BH * L.nqb * sizeof(int));   // query, then key blocks
    L.total = off;
    return L;
}

constexpr int kFusedKernels = 3;
const char *const kFusedNames[kFusedKernels] = {"k_fold", "k_mta_fused", "k_mix_groupnorm"};

// Clusters of the main kernel that fit on the device at once (one CTA per SM
// at this shared-memory size), cached per kernel instantiation and device.
template <int D, int CH>
mta_status max_resident_clusters(const cudaLaunchConfig_t &cfg, int *out)
{
    constexpr bool PAIR = (D == 128);
    constexpr int cluster = PAIR ? 2 : 1;
    auto kernel = k_mta_fused<D, CH, PAIR>;
    constexpr int kMaxDevices = 64;
    static int cached[kMaxDevices] = {};
    static std::mutex lock;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MTA_ERR_CUDA;
    std::lock_guard<std::mutex> guard(lock);
    if (!cached[dev]) {
        int n = 0;
        if (cluster > 1) {
            cudaLaunchConfig_t c = cfg;
            c.gridDim = dim3((unsigned)cluster, 1, 1);
            if (cudaOccupancyMaxActiveClusters(&n, (void *)kernel, &c) != cudaSuccess) return MTA_ERR_CUDA;
        } else {
            int per_sm = 0, sms = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, (int)cfg.blockDim.x,
                                                              cfg.dynamicSmemBytes) != cudaSuccess ||
                cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
                return MTA_ERR_CUDA;
            n = per_sm * sms;
        }
        if (n < 1) return MTA_ERR_CUDA;
        cached[dev] = n;
    }
    *out = cached[dev];
    return MTA_OK;
}

template <int D, int CH>
mta_status launch_fused_t(const mta_shape &s, const ForwardArgs &a, void *ws, cudaStream_t st,
                          const Trace &tr)
{
    constexpr bool PAIR = (D == 128);
    using C = FusedCfg<D, CH, PAIR>;
    const FusedLayout L = fused_layout(s);
    uint8_t *w = (uint8_t *)ws;
    __half *kf = (__half *)(w + L.off_kf);
    __half *qp = (__half *)(w + L.off_qp);
    float *corr = (float *)(w + L.off_corr);
    __half *part = (__half *)(w + L.off_part);
    int *sexp = (int *)(w + L.off_exp);
    const uint64_t BH = (uint64_t)s.B * s.H;
    CUtensorMap mQ, mK, mV;
    {
        uint64_t dims[3] = {(uint64_t)D, (uint64_t)L.nqb * L.NA * 8, BH};
        uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)L.nqb * L.NA * 8 * D * 2};
        uint32_t box[3] = {64, (uint32_t)(L.NA * 8), 1};
        if (!make_tmap_f16(&mQ, qp, 3, dims, strides, box)) return MTA_ERR_CUDA;
    }
    {
        uint64_t dims[3] = {(uint64_t)D, (uint64_t)L.Tp, BH * s.c_q};
        uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)L.Tp * D * 2};
        uint32_t box[3] = {64, (uint32_t)C::kKfRows, 1};
        if (!make_tmap_f16(&mK, kf, 3, dims, strides, box)) return MTA_ERR_CUDA;
    }
    {
        uint64_t dims[3] = {(uint64_t)D, (uint64_t)s.T, BH};
        uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)s.T * D * 2};
        uint32_t box[3] = {64, (uint32_t)kBN, 1};
        if (!make_tmap_bf16(&mV, a.v, 3, dims, strides, box)) return MTA_ERR_CUDA;
    }
    auto main_kernel = k_mta_fused<D, CH, PAIR>;
    const bool ex = a.exact_mask != 0;
    auto fold = s.c_k == 11 ? (ex ? k_fold<D, 11, true> : k_fold<D, 11, false>)
              : s.c_k == 3  ? (ex ? k_fold<D, 3, true> : k_fold<D, 3, false>)
                            : (ex ? k_fold<D, 15, true> : k_fold<D, 15, false>);
    const int pro_smem = (int)prologue_smem_bytes(D);
    if (cudaFuncSetAttribute(main_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(fold, cudaFuncAttributeMaxDynamicSharedMemorySize, pro_smem) !=
            cudaSuccess)
        return MTA_ERR_CUDA;
    const float scale = kLog2e / sqrtf((float)D);
    tr.before(0, st);
    fold<<<dim3((unsigned)(3 * L.nqb * BH)), kProThreads, pro_smem, st>>>(
        (const __nv_bfloat16 *)a.q, (const __nv_bfloat16 *)a.k, a.w_kq, kf, qp, corr, sexp, s.T, L.Tp,
        s.H, L.nqb, s.c_q, s.c_k, scale);
    tr.after(0, st);
    // The main kernel and the GroupNorm kernel are launched with programmatic
    // stream serialisation: each may be scheduled while its predecessor still
    // runs (the predecessor's CTAs signal it), does its set-up, and waits in
    // griddepcontrol.wait until the predecessor has completed and its writes
    // are visible.
    cudaLaunchAttribute pdl;
    pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl.val.programmaticStreamSerializationAllowed = 1;
    tr.before(1, st);
    {
        // persistent: as many clusters as can be resident at once, each
        // walking its share of the work items
        cudaLaunchConfig_t cfg = {};
        cfg.blockDim = dim3(224, 1, 1);
        cfg.dynamicSmemBytes = C::kSmemBytes;
        cfg.stream = st;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = PAIR ? 2 : 1;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1] = pdl;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        const int n_items = (int)BH * (PAIR ? L.nqb / 2 : L.nqb) * C::kSplits;
        int resident = 0;
        if (max_resident_clusters<D, CH>(cfg, &resident) != MTA_OK)
            return MTA_ERR_CUDA;
        const int ncl = resident < n_items ? resident : n_items;
        cfg.gridDim = dim3((unsigned)(ncl * (PAIR ? 2 : 1)), 1, 1);
        if (cudaLaunchKernelEx(&cfg, main_kernel, mQ, mK, mV, (const float *)corr,
                               (const int *)sexp, a.w_head, part,
                               s.T, L.Tp, s.H, s.c_q, L.nqb, (int)BH) != cudaSuccess)
            return MTA_ERR_CUDA;
    }
    tr.after(1, st);
    tr.before(2, st);
    {
        const long long units = (long long)s.B * s.T * s.H;     // (b, t, h)
        const int per_cta = kMixThreads / (D / 8);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)((units + per_cta - 1) / per_cta), 1, 1);
        cfg.blockDim = dim3(kMixThreads, 1, 1);
        cfg.stream = st;
        cfg.attrs = &pdl;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, k_mix_groupnorm<D, CH>, (const __half *)part, a.gn_weight,
                               a.gn_bias, a.depth_scale, a.gate, s.gn_eps,
                               (__nv_bfloat16 *)a.out, s.T, s.H, units) != cudaSuccess)
            return MTA_ERR_CUDA;
    }
    tr.after(2, st);
    return cudaGetLastError() == cudaSuccess ? MTA_OK : MTA_ERR_CUDA;
}

}  // namespace

bool fused_supported(const mta_shape &s)
{
    if (s.io != MTA_BF16) return false;
    if (s.d != 64 && s.d != 128) return false;
    // up to 256 / d output heads per work item; larger groups split in two
    if (!(s.c_h == 1 || s.c_h == 2 || s.c_h == 4 || s.c_h == 8) || s.c_h * s.d > 512) return false;
    if (s.c_q > 8 || s.c_k > 15 || d_m(s.c_q, s.c_k) > kCorrW - 2) return false;
    return true;
}

size_t fused_workspace_bytes(const mta_shape &s) { return fused_layout(s).total; }

int fused_kernel_count(const mta_shape &) { return kFusedKernels; }

const char *fused_kernel_name(const mta_shape &, int index)
{
    return (index >= 0 && index < kFusedKernels) ? kFusedNames[index] : nullptr;
}

mta_status launch_fused(const mta_shape &s, const ForwardArgs &a, void *ws, cudaStream_t st,
                        const Trace &tr)
{
    if (s.d == 128) {
        if (s.c_h == 1) return launch_fused_t<128, 1>(s, a, ws, st, tr);
        if (s.c_h == 2) return launch_fused_t<128, 2>(s, a, ws, st, tr);
        if (s.c_h == 4) return launch_fused_t<128, 4>(s, a, ws, st, tr);
    } else {
        if (s.c_h == 1) return launch_fused_t<64, 1>(s, a, ws, st, tr);
        if (s.c_h == 2) return launch_fused_t<64, 2>(s, a, ws, st, tr);
        if (s.c_h == 4) return launch_fused_t<64, 4>(s, a, ws, st, tr);
        if (s.c_h == 8) return launch_fused_t<64, 8>(s, a, ws, st, tr);
    }
    return MTA_ERR_UNSUPPORTED;
}

mta_status launch_selftest_wait_timeout(long long budget_cycles, cudaStream_t st)
{
    k_selftest_wait_timeout<<<1, 1, 0, st>>>(budget_cycles);
    return cudaGetLastError() == cudaSuccess ? MTA_OK : MTA_ERR_CUDA;
}

// Scratch of mta_forward_noalloc: a file-scope device array, one per device
// that loads the library.  Host code sees only a stand-in symbol; its device
// address is looked up once per device below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[MTA_NOALLOC_SCRATCH_BYTES];

mta_status noalloc_scratch(void **ptr)
{
    constexpr int kMaxDevices = 64;
    struct Entry {
        void *addr;
        unsigned long long ctx;
    };
    static Entry tab[kMaxDevices] = {};
    static std::mutex lock;
    int dev = 0;
    unsigned long long ctx = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MTA_ERR_CUDA;
    if (!current_context_id(&ctx)) return MTA_ERR_CUDA;
    std::lock_guard<std::mutex> guard(lock);
    // the address belongs to the context the module was loaded in: look it up
    // again after the device's context was destroyed and re-created
    if (!tab[dev].addr || tab[dev].ctx != ctx) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return MTA_ERR_CUDA;
        tab[dev].addr = p;
        tab[dev].ctx = ctx;
    }
    *ptr = tab[dev].addr;
    return MTA_OK;
}

// Read and clear of the error word in one atomic step on the caller's
// stream, so that a flag raised between a read and a separate clear is not
// lost; the value goes through a second device word to the host.
__device__ unsigned int g_fused_error_taken;

__global__ void k_take_error() { g_fused_error_taken = atomicExch(&g_fused_error, 0u); }

unsigned int fused_take_error(cudaStream_t st)
{
    k_take_error<<<1, 1, 0, st>>>();
    unsigned int v = 0;
    if (cudaGetLastError() != cudaSuccess ||
        cudaMemcpyFromSymbolAsync(&v, g_fused_error_taken, sizeof(v), 0, cudaMemcpyDeviceToHost,
                                  st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return ~0u;
    return v;
}

}  // namespace mta
