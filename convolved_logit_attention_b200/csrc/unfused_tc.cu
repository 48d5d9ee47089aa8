// Tensor-core kernels of the materialised chain, for bf16 I/O and d = 64 or
// 128: the chain's two dense contractions of "Multi-Token Attention -- Paper
// Graph", section 3.4, on tcgen05 with fp32 accumulation in TMEM.
//
//   k_logits_tc        S1 + S2: map0[i][j] = (j <= i + band) ? q_i . k_j / sqrt(d)
//                      : 0 for one 128 x 128 tile.  Q and K tiles arrive by TMA
//                      (128-byte swizzle), d/16 MMAs (M = N = 128) accumulate
//                      in TMEM, and the fp32 rows leave through a per-warp
//                      staging tile so that every store instruction writes
//                      whole 128-byte row segments.
//   k_pv_groupnorm_tc  S7..S9: out = s_h GroupNorm(A V) for 128 query rows of
//                      one head.  The fp32 rows of A are read, masked to
//                      j <= i, rounded to bf16 and written to shared memory
//                      in the MMA's swizzled K-major layout; V chunks arrive by
//                      TMA (MN-major); O accumulates in TMEM; the GroupNorm of
//                      a row is thread-local (thread = TMEM lane = query row).
//
// Both are bound by HBM: the map is 4 bytes per live logit, written once by
// k_logits_tc and read once by k_pv_groupnorm_tc; the contractions are 2d
// FLOP per logit, a few percent of the tensor pipe at that byte rate.  The
// bf16 products are exact in fp32, so k_logits_tc differs from a CUDA-core
// fp32 dot product only in summation order.  k_pv_groupnorm_tc rounds the
// attention weights to bf16 (8 significant bits), as the fused kernel does
// with its probabilities.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "mta_internal.h"
#include "tc_util.cuh"
#include "tmap.h"

namespace mta {
namespace {

constexpr int kTile = 128;            // query rows of a CTA; key columns of a logit tile
constexpr int kStageStride = 36;      // floats per staged row: 16-B aligned, conflict-free
constexpr int kPvKeys = 64;           // keys per A V chunk (one 128-byte swizzle row)
constexpr int kPvStages = 3;
constexpr int kPvThreads = 256;
constexpr long long kBudget = 1ll << 30;   // cycles per bounded wait (~0.55 s)

// Device error word of these kernels: bit kErrTimeout, a bounded wait
// expired (the same bit as the fused kernels' word).
__device__ unsigned int g_chain_error;
constexpr unsigned int kErrTimeout = 1u;

// Waits for the phase of `bar` with the given parity; gives up when another
// thread of the CTA aborted or after kBudget cycles (then records a timeout
// in the device error word and aborts the CTA).
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity,
                                              volatile int *abort_flag, unsigned int *err)
{
    if (tc::mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (tc::mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > kBudget) {
            *abort_flag = 1;
            atomicOr(err, kErrTimeout);
            return false;
        }
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

// One 128 x 128 tile of map0 per CTA; grid (column tiles, row tiles, B * H),
// 128 threads.  Thread 0 loads and issues; warp w then owns TMEM lanes
// 32w .. 32w+31 (tile rows) for the epilogue.
template <int D>
__global__ void __launch_bounds__(128)
k_logits_tc(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
            float *__restrict__ map0, int T, float scale, int band)
{
    unsigned int *err = &g_chain_error;
    constexpr int kChunks = D / 64;             // 64-element (128-byte) column chunks
    constexpr int kOpBytes = kChunks * 16384;   // one 128-row operand tile
    const int i0 = blockIdx.y * kTile, j0 = blockIdx.x * kTile;
    if (j0 > i0 + kTile - 1 + band) return;     // the whole tile lies past the band
    const int bh = blockIdx.z;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *sQ = base, *sK = base + kOpBytes;
    __shared__ uint64_t bar_load, bar_mma;
    __shared__ uint32_t tslot;
    __shared__ int abort_flag;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar_load, 1);
        tc::mbar_init(&bar_mma, 1);
        abort_flag = 0;
        tc::fence_barrier_init();
    }
    if (warp == 0) { tc::tmem_alloc(&tslot, 128); tc::tmem_relinquish(); }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tm = tslot;
    if (threadIdx.x == 0) {
        tc::mbar_arrive_expect_tx(&bar_load, 2 * kOpBytes);
        for (int c = 0; c < kChunks; ++c) {
            tc::tma_load_3d(sQ + c * 16384, &mapQ, &bar_load, 64 * c, i0, bh);
            tc::tma_load_3d(sK + c * 16384, &mapK, &bar_load, 64 * c, j0, bh);
        }
        if (wait_or_abort(&bar_load, 0, &abort_flag, err)) {
            tc::tc_fence_after();
            const uint32_t idesc = tc::idesc_bf16(kTile, kTile, false, false);
            const uint64_t dq = tc::sdesc_sw128(tc::smem_u32(sQ), 16, 1024);
            const uint64_t dk = tc::sdesc_sw128(tc::smem_u32(sK), 16, 1024);
#pragma unroll
            for (int c = 0; c < kChunks; ++c)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    tc::mma_bf16(tm, dq + (uint64_t)((c * 16384 + kk * 32) >> 4),
                                 dk + (uint64_t)((c * 16384 + kk * 32) >> 4), idesc,
                                 (c | kk) ? 1u : 0u);
            tc::mma_commit(&bar_mma);
        } else {
            // the copies may still land: let them, within a second budget,
            // before the CTA's shared memory is released
            tc::mbar_wait(&bar_load, 0, kBudget);
        }
    }
    const bool ok = __all_sync(0xffffffffu, wait_or_abort(&bar_mma, 0, &abort_flag, err));
    if (ok) {
        tc::tc_fence_after();
        // the operand tiles are dead once the MMAs completed: the staging
        // rows of the four warps (18 KB) reuse them
        float *stage = (float *)base + warp * 32 * kStageStride;
        float *srow = stage + lane * kStageStride;
        const int i = i0 + 32 * warp + lane;
        const bool vec = (T & 3) == 0;
        float *mb = map0 + (size_t)bh * T * T;
#pragma unroll 1
        for (int jc = 0; jc < kTile / 32; ++jc) {
            float s[32];
            tc::tmem_ld32f(tm + ((uint32_t)(32 * warp) << 16) + 32 * jc, s);
            tc::tmem_ld_wait();
            const int jb = j0 + 32 * jc;
#pragma unroll
            for (int c = 0; c < 32; ++c) s[c] = (jb + c <= i + band) ? s[c] * scale : 0.f;
#pragma unroll
            for (int m = 0; m < 8; ++m)
                *reinterpret_cast<float4 *>(srow + 4 * m) =
                    make_float4(s[4 * m], s[4 * m + 1], s[4 * m + 2], s[4 * m + 3]);
            __syncwarp();
            if (vec) {
                // 8 lanes per row: each instruction writes 4 rows x 128 B
#pragma unroll
                for (int rho = 0; rho < 8; ++rho) {
                    const int rr = 4 * rho + (lane >> 3);
                    const int ii = i0 + 32 * warp + rr, jj = jb + 4 * (lane & 7);
                    const float4 v = *reinterpret_cast<const float4 *>(stage + rr * kStageStride +
                                                                       4 * (lane & 7));
                    if (ii < T && jj < T)
                        *reinterpret_cast<float4 *>(mb + (size_t)ii * T + jj) = v;
                }
            } else {
                // rows not 16-byte aligned: one row of 32 floats per instruction
                for (int rr = 0; rr < 32; ++rr) {
                    const int ii = i0 + 32 * warp + rr, jj = jb + lane;
                    if (ii < T && jj < T) mb[(size_t)ii * T + jj] = stage[rr * kStageStride + lane];
                }
            }
            __syncwarp();
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tm, 128);
    }
}

// out rows i0 .. i0+127 of head (b, h): grid (row blocks, B * H), 256
// threads.  Every thread converts its share of each 64-key chunk of A;
// thread 0 also loads V and issues the chunk's MMAs once all threads have
// arrived; stages are recycled when the MMAs that read them have completed.
// Warps 0..3 (TMEM lanes = rows) run the GroupNorm epilogue.
template <int D>
__global__ void __launch_bounds__(kPvThreads, 2)
k_pv_groupnorm_tc(const float *__restrict__ amap, const __grid_constant__ CUtensorMap mapV,
                  const float *__restrict__ gn_weight, const float *__restrict__ gn_bias,
                  float depth_scale, const float *__restrict__ gate, float eps,
                  __nv_bfloat16 *__restrict__ out, int T, int H)
{
    unsigned int *err = &g_chain_error;
    constexpr int kABytes = kTile * kPvKeys * 2;   // 16 KB: 128 rows x 64 keys, bf16
    constexpr int kVBytes = kPvKeys * D * 2;       // 64 keys x D, D/64 chunks of 8 KB
    constexpr int kStageBytes = kABytes + kVBytes;
    // the grid's slow index is the query block, longest first, so the
    // scheduler deals out the causal rows longest-first across the heads
    const int i0 = ((int)gridDim.y - 1 - (int)blockIdx.y) * kTile;
    const int bh = blockIdx.x;
    const int b = bh / H, h = bh % H;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    __shared__ uint64_t a_full[kPvStages], v_full[kPvStages], mma_done[kPvStages];
    __shared__ uint32_t tslot;
    __shared__ int abort_flag;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    if (tid == 0) {
        for (int s = 0; s < kPvStages; ++s) {
            tc::mbar_init(&a_full[s], kPvThreads);
            tc::mbar_init(&v_full[s], 1);
            tc::mbar_init(&mma_done[s], 1);
        }
        abort_flag = 0;
        tc::fence_barrier_init();
    }
    if (warp == 0) { tc::tmem_alloc(&tslot, D); tc::tmem_relinquish(); }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tm = tslot;
    const int jend = min(T, i0 + kTile);          // keys past the block's last row are masked
    const int nch = (jend + kPvKeys - 1) / kPvKeys;
    const bool vec = (T & 3) == 0;
    const float *ab = amap + (size_t)bh * T * T;
    const uint32_t idesc = tc::idesc_bf16(kTile, D, false, true);
    int issued = 0;        // chunks whose V copy thread 0 started
    int committed = 0;     // chunks whose MMAs thread 0 committed
    bool ok = true;
    for (int n = 0; n < nch && ok; ++n) {
        const int s = n % kPvStages;
        const uint32_t use = (uint32_t)(n / kPvStages);
        uint8_t *sA = base + s * kStageBytes;
        uint8_t *sV = sA + kABytes;
        // the stage is free once the MMAs of its previous chunk completed
        if (n >= kPvStages && !wait_or_abort(&mma_done[s], (use - 1) & 1, &abort_flag, err)) {
            ok = false;
            break;
        }
        if (tid == 0) {
            tc::mbar_arrive_expect_tx(&v_full[s], kVBytes);
            for (int c = 0; c < D / 64; ++c)
                tc::tma_load_3d(sV + c * 8192, &mapV, &v_full[s], 64 * c, n * kPvKeys, bh);
            ++issued;
        }
        // A chunk: thread tid takes 16-byte groups f = tid + 256 u: row f / 16,
        // keys 4 (f % 16) .. +3 (a warp reads two 256-byte row segments)
        const int j0 = n * kPvKeys;
        float x[8][4];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int f = tid + kPvThreads * u, r = f >> 4, j = j0 + 4 * (f & 15);
            const int i = i0 + r;
            x[u][0] = x[u][1] = x[u][2] = x[u][3] = 0.f;
            if (i < T && j <= i) {
                const float *src = ab + (size_t)i * T + j;
                if (vec && j + 3 <= i) {
                    const float4 t = __ldg(reinterpret_cast<const float4 *>(src));
                    x[u][0] = t.x; x[u][1] = t.y; x[u][2] = t.z; x[u][3] = t.w;
                } else {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (j + e <= i) x[u][e] = __ldg(src + e);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int f = tid + kPvThreads * u, r = f >> 4, kk = 4 * (f & 15);
            uint2 pk;
            pk.x = pack_bf16x2(x[u][0], x[u][1]);
            pk.y = pack_bf16x2(x[u][2], x[u][3]);
            *reinterpret_cast<uint2 *>(sA + tc::sw128_offset((uint32_t)r, (uint32_t)kk)) = pk;
        }
        tc::fence_async_shared();
        tc::mbar_arrive(&a_full[s]);
        if (tid == 0) {
            if (!wait_or_abort(&a_full[s], use & 1, &abort_flag, err) ||
                !wait_or_abort(&v_full[s], use & 1, &abort_flag, err)) {
                ok = false;
                break;
            }
            tc::tc_fence_after();
            const uint64_t da = tc::sdesc_sw128(tc::smem_u32(sA), 16, 1024);
            const uint64_t dv = tc::sdesc_sw128(tc::smem_u32(sV), 8192, 1024);
#pragma unroll
            for (int kk = 0; kk < kPvKeys / 16; ++kk)
                tc::mma_bf16(tm, da + (uint64_t)((kk * 32) >> 4), dv + (uint64_t)((kk * 2048) >> 4),
                             idesc, (n | kk) ? 1u : 0u);
            tc::mma_commit(&mma_done[s]);
            ++committed;
        }
    }
    // the last commit covers every MMA of the block
    const int last = nch - 1;
    ok = ok && wait_or_abort(&mma_done[last % kPvStages], (uint32_t)(last / kPvStages) & 1,
                             &abort_flag, err);
    if (tid == 0 && !ok) {
        // after an abort: let this thread's copies and MMAs in flight finish
        // (bounded) before shared memory and TMEM are released
        for (int n = (issued > kPvStages ? issued - kPvStages : 0); n < issued; ++n)
            tc::mbar_wait(&v_full[n % kPvStages], (uint32_t)(n / kPvStages) & 1, kBudget);
        if (committed > 0)
            tc::mbar_wait(&mma_done[(committed - 1) % kPvStages],
                          (uint32_t)((committed - 1) / kPvStages) & 1, kBudget);
    }
    if (warp < 4 && __all_sync(0xffffffffu, ok)) {
        tc::tc_fence_after();
        const int i = i0 + 32 * warp + lane;
        const uint32_t row = tm + ((uint32_t)(32 * warp) << 16);
        // GroupNorm over the row's D channels in three passes over TMEM
        // (mean, centred second moment, output), 32 columns at a time
        float v[32];
        float sum = 0.f;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
            tc::tmem_ld32f(row + 32 * c, v);
            tc::tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) sum += v[e];
        }
        const float mean = sum / D;
        float s2 = 0.f;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
            tc::tmem_ld32f(row + 32 * c, v);
            tc::tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) { const float t = v[e] - mean; s2 += t * t; }
        }
        const float inv = 1.f / sqrtf(s2 / D + eps);
        const float sc = gate ? 1.f / (1.f + expf(-gate[h])) : depth_scale;
        __nv_bfloat16 *dst = out + ((size_t)b * T + i) * ((size_t)H * D) + (size_t)h * D;
        const float *gw = gn_weight + (size_t)h * D, *gb = gn_bias + (size_t)h * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
            tc::tmem_ld32f(row + 32 * c, v);
            tc::tmem_ld_wait();
            if (i < T) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint4 w;
                    uint32_t *wp = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const int e = 8 * q + 2 * p, ch = 32 * c + e;
                        wp[p] = pack_bf16x2(sc * ((v[e] - mean) * inv * gw[ch] + gb[ch]),
                                            sc * ((v[e + 1] - mean) * inv * gw[ch + 1] + gb[ch + 1]));
                    }
                    *reinterpret_cast<uint4 *>(dst + 32 * c + 8 * q) = w;
                }
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tm, D);
    }
}

// ----------------------------------------------------------------------------
// fp32 products on tensor cores (3xTF32) for the backward pass.
//
// A TF32 operand keeps sign, exponent and the top 10 mantissa bits of an fp32
// word.  With x_hi = x with its low 13 mantissa bits cleared (exact in TF32)
// and x_lo = x - x_hi (exact in fp32, at most 2^-10 |x|),
//   A B = A_hi B_hi + A_lo B_hi + A_hi B_lo + A_lo B_lo,
// and the last term (at most 2^-20 |A B| per product) is dropped; x_lo itself
// enters the MMA with a further relative error of 2^-10 at most, so every
// product carries about 2^-20 relative error before the fp32 accumulation:
// the accuracy of an fp32 dot product, at tensor-core rate (three TF32 MMAs
// per K step, two when the X operand is bf16, whose x_lo is 0).
//
// k_mm_tf32<MODE, D, TX>, one 128-row block of output per CTA, 256 threads,
// contraction in chunks of 32 (one 128-byte swizzled row of fp32):
//   MODE 0: out[r][e] = scale * sum_{j <= r} map[r][j] X[j][e]     (O = A V, dQ)
//   MODE 1: out[r][e] = scale * sum_{i >= r} map[i][r] X[i][e]     (dV = A^T dO, dK)
//   MODE 2: map[i][j] = scale * sum_e A[i][e] X[j][e] for j <= i, 0 above,
//           one 128 x 128 tile of the causal triangle               (dA = dO V^T)
// The raw source rows of a chunk are copied with cp.async into a ring of
// staging buffers, one chunk ahead; each copy's completion is counted on the
// buffer's barrier (one arrival per thread).  Every thread then converts its
// share of the chunk from shared memory into the K-major hi and lo tiles in
// the MMA's 128-byte-swizzled layout (transposed where the source runs along
// the tile's rows, masked to the causal triangle), and thread 0 issues the
// chunk's MMAs once all threads have arrived; their commit frees the tiles for
// the next chunk.  Rows of the map must be 16-byte aligned (T % 4 == 0).
constexpr int kMmKc = 32;             // contraction indices per chunk

__device__ __forceinline__ float tf32_hi(float x)
{
    return __uint_as_float(__float_as_uint(x) & 0xffffe000u);
}

// Byte offset of fp32 element (row, k) of a K-major 128-byte-swizzled tile
// whose rows hold 32 elements (tile base 1024-byte aligned).
__device__ __forceinline__ uint32_t sw128_f32(uint32_t row, uint32_t k)
{
    return row * 128u + ((((k >> 2) ^ (row & 7u)) & 7u) << 4) + ((k & 3u) << 2);
}

// Transposed conversion (a source that runs along the tile's rows, read for 32
// contraction indices): slot = warp + 8u and lane give contraction index
// tq_k and row quad tq_q (rows 4 tq_q .. +3).  A warp reads 16 staged rows x
// 32 bytes and each of its four scalar stores per quad hits 32 distinct banks
// of the K-major swizzled tile.
__device__ __forceinline__ int tq_k(int slot, int lane) { return 16 * (slot & 1) + (lane & 15); }
__device__ __forceinline__ int tq_q(int slot, int lane) { return 2 * (slot >> 1) + (lane >> 4); }

__device__ __forceinline__ void store_split4(uint8_t *hi, uint8_t *lo, uint32_t off, float4 v)
{
    const float4 h = make_float4(tf32_hi(v.x), tf32_hi(v.y), tf32_hi(v.z), tf32_hi(v.w));
    *reinterpret_cast<float4 *>(hi + off) = h;
    *reinterpret_cast<float4 *>(lo + off) = make_float4(v.x - h.x, v.y - h.y, v.z - h.z, v.w - h.w);
}

__device__ __forceinline__ void store_split1(uint8_t *hi, uint8_t *lo, uint32_t off, float v)
{
    const float h = tf32_hi(v);
    *reinterpret_cast<float *>(hi + off) = h;
    *reinterpret_cast<float *>(lo + off) = v - h;
}

__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 ld4(const __nv_bfloat16 *p)
{
    const uint2 t = *reinterpret_cast<const uint2 *>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162 *>(&t.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&t.y);
    return make_float4(__low2float(a), __high2float(a), __low2float(b), __high2float(b));
}

template <int MODE, int D, typename TX>
struct MmCfg {
    static constexpr bool kXlo = sizeof(TX) == 4;               // an fp32 X operand has a lo part
    static constexpr int kES = (int)sizeof(TX);
    static constexpr int N = MODE == 2 ? kTile : D;             // accumulator columns
    static constexpr int kATile = kTile * kMmKc * 4;            // 16 KB
    static constexpr int kBTile = N * kMmKc * 4;
    static constexpr int kStage = 2 * kATile + (kXlo ? 2 : 1) * kBTile;
    // staging: the A rows (MODE 1: 32 map rows of 128 keys, padded by 16 B so
    // that transposed reads spread over the banks) and the X rows (MODE 0/1:
    // 32 rows of D, padded; MODE 2: 128 rows of 32 channels)
    static constexpr int kAPitch = MODE == 1 ? kTile * 4 + 16 : kMmKc * 4;       // bytes
    static constexpr int kARows = MODE == 1 ? kMmKc : kTile;
    static constexpr int kXPitch = MODE == 2 ? kMmKc * kES : D * kES + 16;
    static constexpr int kXRows = MODE == 2 ? kTile : kMmKc;
    static constexpr int kRawA = kARows * kAPitch;
    static constexpr int kRaw = (kRawA + kXRows * kXPitch + 1023) / 1024 * 1024;
    // one tile stage and two staging buffers: 97 KB with a bf16 X, so two CTAs
    // share an SM and one's conversion, MMAs and stores overlap the other's
    // (measured faster than two tile stages and three staging buffers at one
    // CTA per SM); 130 KB, one CTA per SM, with an fp32 X
    static constexpr int kStages = 1;
    static constexpr int kRawStages = 2;
    static constexpr int kSmem = kStages * kStage + kRawStages * kRaw + 1024;
    static constexpr int kMinBlocks = kSmem <= 113 * 1024 ? 2 : 1;
    static_assert(kSmem <= 227 * 1024, "shared memory");
    static constexpr int kACopies = kARows * kAPitch / 16 / kPvThreads;   // 16-B copies per thread
    static constexpr int kXCopies = kXRows * (MODE == 2 ? kMmKc * kES : D * kES) / 16 / kPvThreads;
    static constexpr int kBU = N * kMmKc / 4 / kPvThreads;     // X groups of 4 per thread
};

template <int MODE, int D, typename TX>
__global__ void __launch_bounds__(kPvThreads, MmCfg<MODE, D, TX>::kMinBlocks)
k_mm_tf32(const float *__restrict__ asrc, const TX *__restrict__ x, float *__restrict__ out, int T,
          float scale)
{
    using C = MmCfg<MODE, D, TX>;
    constexpr int R = C::kRawStages;
    unsigned int *err = &g_chain_error;
    int r0, j0 = 0, c_begin, c_end;
    const int bh = MODE == 2 ? blockIdx.z : blockIdx.x;
    if (MODE == 2) {
        r0 = blockIdx.y * kTile;
        j0 = blockIdx.x * kTile;
        if (j0 > r0 + kTile - 1) return;                         // the tile lies above the diagonal
        c_begin = 0;
        c_end = D;
    } else {
        // longest contraction first (the row block is the grid's slow index, so
        // the order holds across the heads): MODE 0 grows with the row block,
        // MODE 1 shrinks
        const int blk = MODE == 0 ? (int)gridDim.y - 1 - (int)blockIdx.y : (int)blockIdx.y;
        r0 = blk * kTile;
        c_begin = MODE == 0 ? 0 : r0;
        c_end = MODE == 0 ? min(T, r0 + kTile) : T;
    }
    const int nch = (c_end - c_begin + kMmKc - 1) / kMmKc;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *raw0 = base + C::kStages * C::kStage;
    __shared__ uint64_t a_full[C::kStages], mma_done[C::kStages], raw_full[C::kRawStages];
    __shared__ uint32_t tslot;
    __shared__ int abort_flag;
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    if (tid == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            tc::mbar_init(&a_full[s], kPvThreads);
            tc::mbar_init(&mma_done[s], 1);
        }
        for (int s = 0; s < R; ++s) tc::mbar_init(&raw_full[s], kPvThreads);
        abort_flag = 0;
        tc::fence_barrier_init();
    }
    if (warp == 0) { tc::tmem_alloc(&tslot, C::N); tc::tmem_relinquish(); }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tm = tslot;
    const size_t TT = (size_t)T * T;
    const float *amap = asrc + (size_t)bh * (MODE == 2 ? (size_t)T * D : TT);
    const TX *xb = x + (size_t)bh * T * D;
    // cp.async of chunk n into raw stage n % R (rows outside [0, T) zero-filled)
    auto issue_copies = [&](int n) {
        uint8_t *ra = raw0 + (n % R) * C::kRaw;
        uint8_t *rx = ra + C::kRawA;
        const int c0 = c_begin + n * kMmKc;
#pragma unroll
        for (int u = 0; u < C::kACopies; ++u) {
            const int f = tid + kPvThreads * u;
            if (MODE == 1) {                 // map row c0 + (f >> 5), keys r0 + 4 (f & 31) .. +3
                const int i = c0 + (f >> 5), j = r0 + 4 * (f & 31);
                const bool in = i < T && j < T;
                tc::cp_async16(ra + (f >> 5) * C::kAPitch + 16 * (f & 31),
                               amap + (in ? (size_t)i * T + j : 0), in);
            } else if (MODE == 0) {          // map row r0 + (f >> 3), keys c0 + 4 (f & 7) .. +3
                const int i = r0 + (f >> 3), j = c0 + 4 * (f & 7);
                const bool in = i < T && j < T;
                tc::cp_async16(ra + (f >> 3) * C::kAPitch + 16 * (f & 7),
                               amap + (in ? (size_t)i * T + j : 0), in);
            } else {                         // A row r0 + (f >> 3), channels c0 + 4 (f & 7) .. +3
                const int i = r0 + (f >> 3);
                const bool in = i < T;
                tc::cp_async16(ra + (f >> 3) * C::kAPitch + 16 * (f & 7),
                               amap + (in ? (size_t)i * D + c0 + 4 * (f & 7) : 0), in);
            }
        }
        constexpr int kRowChunks = (MODE == 2 ? kMmKc * C::kES : D * C::kES) / 16;
#pragma unroll
        for (int u = 0; u < C::kXCopies; ++u) {
            const int f = tid + kPvThreads * u, row = f / kRowChunks, q = f % kRowChunks;
            const int g = MODE == 2 ? j0 + row : c0 + row;           // source row of X
            const bool in = g < T;
            const uint8_t *src = reinterpret_cast<const uint8_t *>(xb) +
                                 (in ? (size_t)g * D * C::kES + (MODE == 2 ? (size_t)c0 * C::kES : 0) : 0) +
                                 16 * q;
            tc::cp_async16(rx + row * C::kXPitch + 16 * q, src, in);
        }
        tc::cp_async_mbar_arrive(&raw_full[n % R]);
    };
    // chunk n from raw stage n % R into the hi / lo tiles of stage st
    auto convert = [&](int n, uint8_t *st) {
        const uint8_t *ra = raw0 + (n % R) * C::kRaw;
        const uint8_t *rx = ra + C::kRawA;
        const int c0 = c_begin + n * kMmKc;
        uint8_t *ahi = st, *alo = st + C::kATile;
        uint8_t *bhi = st + 2 * C::kATile, *blo = bhi + C::kBTile;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (MODE == 1) {                 // transposed: rows (keys) 4 tq_q + q, column tq_k
                const int slot = warp + 8 * u, kk = tq_k(slot, lane), rr = 4 * tq_q(slot, lane);
                const float4 v = *reinterpret_cast<const float4 *>(ra + kk * C::kAPitch + 4 * rr);
                const int i = c0 + kk, j = r0 + rr;
                const float w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    store_split1(ahi, alo, sw128_f32(rr + q, kk),
                                 (i < T && j + q <= i) ? w[q] : 0.f);
            } else {
                const int f = tid + kPvThreads * u, row = f >> 3, k4 = 4 * (f & 7);
                float4 v = *reinterpret_cast<const float4 *>(ra + row * C::kAPitch + 4 * k4);
                if (MODE == 0) {             // the causal mask (the map holds garbage above it)
                    const int i = r0 + row, j = c0 + k4;
                    v.x = j <= i ? v.x : 0.f;
                    v.y = j + 1 <= i ? v.y : 0.f;
                    v.z = j + 2 <= i ? v.z : 0.f;
                    v.w = j + 3 <= i ? v.w : 0.f;
                }
                store_split4(ahi, alo, sw128_f32(row, k4), v);
            }
        }
#pragma unroll
        for (int u = 0; u < C::kBU; ++u) {
            if (MODE == 2) {
                const int f = tid + kPvThreads * u, row = f >> 3, k4 = 4 * (f & 7);
                const float4 v = ld4(reinterpret_cast<const TX *>(rx + row * C::kXPitch) + k4);
                const uint32_t off = sw128_f32(row, k4);
                if (C::kXlo) store_split4(bhi, blo, off, v);
                else *reinterpret_cast<float4 *>(bhi + off) = v;    // bf16 values are exact in TF32
            } else {                         // transposed: rows (channels) 4 tq_q + q, column tq_k
                const int slot = warp + 8 * u, kk = tq_k(slot, lane), e = 4 * tq_q(slot, lane);
                const float4 v = ld4(reinterpret_cast<const TX *>(rx + kk * C::kXPitch) + e);
                const float w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t off = sw128_f32(e + q, kk);
                    if (C::kXlo) store_split1(bhi, blo, off, w[q]);
                    else *reinterpret_cast<float *>(bhi + off) = w[q];
                }
            }
        }
    };
    const uint32_t idesc = tc::idesc_tf32(kTile, C::N, false, false);
    int committed = 0;
    bool ok = true;
    for (int p = 0; p < R && p < nch; ++p) issue_copies(p);
    for (int n = 0; n < nch && ok; ++n) {
        const int s = n % C::kStages;
        const uint32_t use = (uint32_t)(n / C::kStages);
        uint8_t *st = base + s * C::kStage;
        if (!wait_or_abort(&raw_full[n % R], (uint32_t)(n / R) & 1, &abort_flag, err)) {
            ok = false;
            break;
        }
        if (n >= C::kStages && !wait_or_abort(&mma_done[s], (use - 1) & 1, &abort_flag, err)) {
            ok = false;
            break;
        }
        convert(n, st);
        tc::fence_async_shared();
        tc::mbar_arrive(&a_full[s]);
        // every thread has converted chunk n once a_full completes: its raw
        // stage takes chunk n + R, and thread 0 issues chunk n's MMAs
        if (!wait_or_abort(&a_full[s], use & 1, &abort_flag, err)) {
            ok = false;
            break;
        }
        if (tid == 0) {
            tc::tc_fence_after();
            const uint64_t dah = tc::sdesc_sw128(tc::smem_u32(st), 16, 1024);
            const uint64_t dal = tc::sdesc_sw128(tc::smem_u32(st + C::kATile), 16, 1024);
            const uint64_t dbh = tc::sdesc_sw128(tc::smem_u32(st + 2 * C::kATile), 16, 1024);
            const uint64_t dbl = tc::sdesc_sw128(tc::smem_u32(st + 2 * C::kATile + C::kBTile), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < kMmKc / 8; ++kk) {       // K = 8 per MMA: 32 bytes of a row
                const uint64_t o = (uint64_t)((kk * 32) >> 4);
                tc::mma_tf32(tm, dah + o, dbh + o, idesc, (n | kk) ? 1u : 0u);
                tc::mma_tf32(tm, dal + o, dbh + o, idesc, 1u);
                if (C::kXlo) tc::mma_tf32(tm, dah + o, dbl + o, idesc, 1u);
            }
            tc::mma_commit(&mma_done[s]);
            ++committed;
        }
        if (n + R < nch) issue_copies(n + R);
    }
    const int last = nch - 1;
    ok = ok && wait_or_abort(&mma_done[last % C::kStages], (uint32_t)(last / C::kStages) & 1,
                             &abort_flag, err);
    tc::cp_async_wait_all();                // no copy of this thread is still in flight
    if (tid == 0 && !ok && committed > 0)   // after an abort: the MMAs in flight finish first
        tc::mbar_wait(&mma_done[(committed - 1) % C::kStages],
                      (uint32_t)((committed - 1) / C::kStages) & 1, kBudget);
    if (warp < 4 && __all_sync(0xffffffffu, ok)) {
        tc::tc_fence_after();
        const int i = r0 + 32 * warp + lane;
        const uint32_t row = tm + ((uint32_t)(32 * warp) << 16);
        if (MODE != 2) {
            float *dst = out + ((size_t)bh * T + i) * D;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                float v[32];
                tc::tmem_ld32f(row + 32 * c, v);
                tc::tmem_ld_wait();
                if (i < T) {
#pragma unroll
                    for (int m = 0; m < 8; ++m)
                        *reinterpret_cast<float4 *>(dst + 32 * c + 4 * m) =
                            make_float4(v[4 * m] * scale, v[4 * m + 1] * scale, v[4 * m + 2] * scale,
                                        v[4 * m + 3] * scale);
                }
            }
        } else {
            // the map tile, through a per-warp staging tile (stage 0 is free:
            // every MMA has completed) so that stores cover whole row segments
            float *stage = (float *)base + warp * 32 * kStageStride;
            float *srow = stage + lane * kStageStride;
            float *mb = out + (size_t)bh * TT;
#pragma unroll 1
            for (int jc = 0; jc < kTile / 32; ++jc) {
                float v[32];
                tc::tmem_ld32f(row + 32 * jc, v);
                tc::tmem_ld_wait();
                const int jb = j0 + 32 * jc;
#pragma unroll
                for (int c = 0; c < 32; ++c) v[c] = (jb + c <= i) ? v[c] * scale : 0.f;
#pragma unroll
                for (int m = 0; m < 8; ++m)
                    *reinterpret_cast<float4 *>(srow + 4 * m) =
                        make_float4(v[4 * m], v[4 * m + 1], v[4 * m + 2], v[4 * m + 3]);
                __syncwarp();
#pragma unroll
                for (int rho = 0; rho < 8; ++rho) {
                    const int rr = 4 * rho + (lane >> 3);
                    const int ii = r0 + 32 * warp + rr, jj = jb + 4 * (lane & 7);
                    const float4 t = *reinterpret_cast<const float4 *>(stage + rr * kStageStride +
                                                                       4 * (lane & 7));
                    if (ii < T && jj < T) *reinterpret_cast<float4 *>(mb + (size_t)ii * T + jj) = t;
                }
                __syncwarp();
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tm, C::N);
    }
}

template <int MODE, int D, typename TX>
mta_status launch_mm_tf32_t(const mta_shape &s, const float *a, const void *xv, float *out,
                            float scale, cudaStream_t st)
{
    using C = MmCfg<MODE, D, TX>;
    auto kern = k_mm_tf32<MODE, D, TX>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem) !=
        cudaSuccess)
        return MTA_ERR_CUDA;
    const int nb = (s.T + kTile - 1) / kTile;
    const unsigned BH = (unsigned)(s.B * s.H);
    const dim3 grid = MODE == 2 ? dim3(nb, nb, BH) : dim3(BH, nb);
    kern<<<grid, kPvThreads, C::kSmem, st>>>(a, (const TX *)xv, out, s.T, scale);
    return cudaGetLastError() == cudaSuccess ? MTA_OK : MTA_ERR_CUDA;
}

template <int MODE, typename TX>
mta_status launch_mm_tf32_d(const mta_shape &s, const float *a, const void *xv, float *out,
                            float scale, cudaStream_t st)
{
    return s.d == 128 ? launch_mm_tf32_t<MODE, 128, TX>(s, a, xv, out, scale, st)
                      : launch_mm_tf32_t<MODE, 64, TX>(s, a, xv, out, scale, st);
}

template <int MODE>
mta_status launch_mm_tf32(const mta_shape &s, const float *a, const void *xv, bool x_io,
                          float *out, float scale, cudaStream_t st)
{
    if (x_io && s.io == MTA_BF16)
        return launch_mm_tf32_d<MODE, __nv_bfloat16>(s, a, xv, out, scale, st);
    return launch_mm_tf32_d<MODE, float>(s, a, xv, out, scale, st);
}

template <int D>
mta_status launch_logits_tc_t(const mta_shape &s, const void *q, const void *k, float *map0,
                              int band, cudaStream_t st)
{
    const uint64_t BH = (uint64_t)s.B * s.H;
    CUtensorMap mQ, mK;
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)s.T, BH};
    const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)s.T * D * 2};
    const uint32_t box[3] = {64, (uint32_t)kTile, 1};
    if (!make_tmap_bf16(&mQ, q, 3, dims, strides, box) ||
        !make_tmap_bf16(&mK, k, 3, dims, strides, box))
        return MTA_ERR_CUDA;
    // at d = 64 the operands take 33 KB; the request is raised so that at
    // most four CTAs (4 x 128 TMEM columns) share an SM and no allocation waits
    const int smem = 2 * (D / 64) * 16384 + 1024 > 50 * 1024 ? 2 * (D / 64) * 16384 + 1024
                                                              : 50 * 1024;
    if (cudaFuncSetAttribute(k_logits_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
        return MTA_ERR_CUDA;
    const int nt = (s.T + kTile - 1) / kTile;
    k_logits_tc<D><<<dim3(nt, nt, (unsigned)BH), 128, smem, st>>>(
        mQ, mK, map0, s.T, 1.0f / sqrtf((float)D), band);
    return cudaGetLastError() == cudaSuccess ? MTA_OK : MTA_ERR_CUDA;
}

template <int D>
mta_status launch_pv_tc_t(const mta_shape &s, const float *amap, const ForwardArgs &a,
                          cudaStream_t st)
{
    const uint64_t BH = (uint64_t)s.B * s.H;
    CUtensorMap mV;
    const uint64_t dims[3] = {(uint64_t)D, (uint64_t)s.T, BH};
    const uint64_t strides[2] = {(uint64_t)D * 2, (uint64_t)s.T * D * 2};
    const uint32_t box[3] = {64, (uint32_t)kPvKeys, 1};
    if (!make_tmap_bf16(&mV, a.v, 3, dims, strides, box)) return MTA_ERR_CUDA;
    const int smem = kPvStages * (kTile * kPvKeys * 2 + kPvKeys * D * 2) + 1024;
    if (cudaFuncSetAttribute(k_pv_groupnorm_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem) != cudaSuccess)
        return MTA_ERR_CUDA;
    const int nb = (s.T + kTile - 1) / kTile;
    k_pv_groupnorm_tc<D><<<dim3((unsigned)BH, nb), kPvThreads, smem, st>>>(
        amap, mV, a.gn_weight, a.gn_bias, a.depth_scale, a.gate, s.gn_eps,
        (__nv_bfloat16 *)a.out, s.T, s.H);
    return cudaGetLastError() == cudaSuccess ? MTA_OK : MTA_ERR_CUDA;
}

__device__ unsigned int g_chain_error_taken;

__global__ void k_take_chain_error() { g_chain_error_taken = atomicExch(&g_chain_error, 0u); }

}  // namespace

unsigned int chain_take_error(cudaStream_t st)
{
    k_take_chain_error<<<1, 1, 0, st>>>();
    unsigned int v = 0;
    if (cudaGetLastError() != cudaSuccess ||
        cudaMemcpyFromSymbolAsync(&v, g_chain_error_taken, sizeof(v), 0, cudaMemcpyDeviceToHost,
                                  st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return ~0u;
    return v;
}

bool mm_tf32_supported(const mta_shape &s)
{
    return (s.d == 64 || s.d == 128) && s.T % 4 == 0;   // 16-byte map rows for cp.async
}

mta_status causal_mm_tf32(const mta_shape &s, bool trans, const float *map, const void *x,
                          bool x_io, float *out, float scale, cudaStream_t st)
{
    return trans ? launch_mm_tf32<1>(s, map, x, x_io, out, scale, st)
                 : launch_mm_tf32<0>(s, map, x, x_io, out, scale, st);
}

mta_status logits_f32_tf32(const mta_shape &s, const float *a, const void *b, float scale,
                           float *map, cudaStream_t st)
{
    return launch_mm_tf32<2>(s, a, b, true, map, scale, st);
}

bool chain_tc_supported(const mta_shape &s)
{
    return s.io == MTA_BF16 && (s.d == 64 || s.d == 128);
}

mta_status logits_tc(const mta_shape &s, const void *q, const void *k, float *map0, int band,
                     cudaStream_t st)
{
    return s.d == 128 ? launch_logits_tc_t<128>(s, q, k, map0, band, st)
                      : launch_logits_tc_t<64>(s, q, k, map0, band, st);
}

mta_status pv_groupnorm_tc(const mta_shape &s, const float *amap, const ForwardArgs &a,
                           cudaStream_t st)
{
    return s.d == 128 ? launch_pv_tc_t<128>(s, amap, a, st) : launch_pv_tc_t<64>(s, amap, a, st);
}

}  // namespace mta
