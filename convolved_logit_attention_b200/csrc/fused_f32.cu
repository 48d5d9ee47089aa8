// Fused MTA forward for fp32 I/O on CUDA cores (FFMA), with no T x T map in
// HBM.  fp16 tensor-core operands (the bf16 path's k_mta_fused) cannot meet
// the fp32 tolerance, so this kernel computes every step of "Multi-Token
// Attention -- Paper Graph", section 3.4, in fp32:
//
//   k_mta_fused_f32  one CTA per (b, head group g, 16 query rows i0 ..).
//     For every key tile of 32 keys j0 .. j0+31 up to the diagonal:
//       - the masked logits A0[r][c] = q_r . k_c / sqrt(d) (Mask_0: zero for
//         c > r, and zero outside [0,T)) of the rows r = i0 - c_q + 1 .. i0+15
//         and keys c = j0 - ceil(c_k/2) + 1 .. j0 + 31 + floor(c_k/2) that the
//         tile's convolution reads, for the c_h heads of the group, in shared
//         memory;
//       - the Eq. (4) convolution C[i][j] with Mask_-inf for j > i.
//     Pass 1 keeps each (row, head)'s running max and sum of exp; pass 2
//     recomputes the tiles, forms P = exp(C - m) / l, the Eq. (7) head mix
//     A^h = sum_h' w[h][h'] P^h', and accumulates O^h += A^h V^h.
//     Epilogue: GroupNorm over each head's d values, affine, and the depth
//     scale or sigmoid(g_h).
// Shapes with c_h * d <= 256 (every shape of the fp32 workloads) take it.
#include <cuda_runtime.h>
#include <math.h>

#include "mta_internal.h"

namespace mta {
namespace {

constexpr int kRB = 16;          // query rows per CTA
constexpr int kKT = 32;          // keys per tile
constexpr int kMaxCq = 8, kMaxCk = 15, kMaxD = 128;
constexpr int kMaxCHD = 256;     // c_h * d
constexpr int kRowsA = kRB + kMaxCq - 1;       // logit rows of a tile
constexpr int kKeysA = kKT + kMaxCk - 1;       // logit keys of a tile
constexpr int kThreads = 256;

struct F32Smem {
    float q[kRowsA * kMaxCHD];          // [head][row][e] (rows i0 - c_q + 1 ..)
    float kv[kKeysA * kMaxCHD];         // k rows of the tile, then v rows
    float a0[16 * kRowsA * kKeysA];     // [head][row][key], c_h <= 16
    float c[16 * kRB * kKT];            // [head][row][key], c_h <= 16
    float o[kRB * kMaxCHD];             // [row][head][e]
    float m[16 * kRB], l[16 * kRB];     // [head][row]
    float th[16 * kMaxCq * 16];         // taps [head][i'][j'] padded to 16
    float w[16 * 16];
};

__global__ void __launch_bounds__(kThreads)
k_mta_fused_f32(const float *__restrict__ q, const float *__restrict__ k,
                const float *__restrict__ v, const float *__restrict__ w_kq,
                const float *__restrict__ w_head, const float *__restrict__ gn_weight,
                const float *__restrict__ gn_bias, float depth_scale,
                const float *__restrict__ gate, float eps, float *__restrict__ out, int T, int H,
                int d, int c_q, int c_k, int c_h)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    F32Smem &S = *reinterpret_cast<F32Smem *>(smem_raw);
    const int i0 = blockIdx.x * kRB;
    const int G = H / c_h;
    const int b = blockIdx.y / G, g = blockIdx.y % G;
    const int tid = threadIdx.x;
    const int rows = kRB + c_q - 1;
    const int Lk = (c_k + 1) / 2 - 1;            // keys reached to the left of a tile
    const int keys = kKT + c_k - 1;
    const float rsd = 1.f / sqrtf((float)d);
    const size_t head0 = (size_t)b * H + (size_t)g * c_h;   // first (b, h) of the group

    for (int idx = tid; idx < c_h * c_q * 16; idx += kThreads) {
        const int hh = idx / (c_q * 16), ip = (idx / 16) % c_q, jj = idx % 16;
        S.th[(hh * kMaxCq + ip) * 16 + jj] =
            jj < c_k ? w_kq[(((size_t)g * c_h + hh) * c_q + ip) * c_k + jj] : 0.f;
    }
    for (int idx = tid; idx < c_h * c_h; idx += kThreads) S.w[idx] = w_head[(size_t)g * c_h * c_h + idx];
    // the query rows i0 - c_q + 1 .. i0 + 15 of every head (zero outside [0,T))
    for (int idx = tid; idx < c_h * rows * d; idx += kThreads) {
        const int hh = idx / (rows * d), rr = (idx / d) % rows, e = idx % d;
        const int r = i0 - (c_q - 1) + rr;
        S.q[(hh * kRowsA + rr) * d + e] =
            (r >= 0 && r < T) ? q[((head0 + hh) * T + r) * (size_t)d + e] : 0.f;
    }
    for (int idx = tid; idx < kRB * c_h * d; idx += kThreads) S.o[idx] = 0.f;
    for (int idx = tid; idx < c_h * kRB; idx += kThreads) { S.m[idx] = -INFINITY; S.l[idx] = 0.f; }
    __syncthreads();

    const int last_key = min(T - 1, i0 + kRB - 1);
    for (int pass = 0; pass < 2; ++pass) {
        for (int j0 = 0; j0 <= last_key; j0 += kKT) {
            // k rows of the tile's logits: keys j0 - Lk .. j0 - Lk + keys - 1
            for (int idx = tid; idx < c_h * keys * d; idx += kThreads) {
                const int hh = idx / (keys * d), cc = (idx / d) % keys, e = idx % d;
                const int c = j0 - Lk + cc;
                S.kv[(hh * kKeysA + cc) * d + e] =
                    (c >= 0 && c < T) ? k[((head0 + hh) * T + c) * (size_t)d + e] : 0.f;
            }
            __syncthreads();
            // masked logits A0[head][rr][cc], rows r = i0 - c_q + 1 + rr, keys c
            for (int idx = tid; idx < c_h * rows * keys; idx += kThreads) {
                const int hh = idx / (rows * keys), rr = (idx / keys) % rows, cc = idx % keys;
                const int r = i0 - (c_q - 1) + rr, c = j0 - Lk + cc;
                float a = 0.f;
                if (r >= 0 && r < T && c >= 0 && c <= r) {
                    const float *qr = S.q + (hh * kRowsA + rr) * d;
                    const float *kc = S.kv + (hh * kKeysA + cc) * d;
                    for (int e = 0; e < d; ++e) a = fmaf(qr[e], kc[e], a);
                    a *= rsd;
                }
                S.a0[(hh * kRowsA + rr) * kKeysA + cc] = a;
            }
            __syncthreads();
            // the Eq. (4) convolution and Mask_-inf: output (i0 + ro, j0 + co),
            // tap (i', jj) reads A0 row ro + c_q - 1 - i', key co + c_k - 1 - jj
            for (int idx = tid; idx < c_h * kRB * kKT; idx += kThreads) {
                const int hh = idx / (kRB * kKT), ro = (idx / kKT) % kRB, co = idx % kKT;
                const int i = i0 + ro, j = j0 + co;
                float cval = -INFINITY;
                if (i < T && j <= i) {
                    cval = 0.f;
                    for (int ip = 0; ip < c_q; ++ip) {
                        const float *arow = S.a0 + (hh * kRowsA + ro + c_q - 1 - ip) * kKeysA + co + c_k - 1;
                        const float *tr = S.th + (hh * kMaxCq + ip) * 16;
                        for (int jj = 0; jj < c_k; ++jj) cval = fmaf(tr[jj], arow[-jj], cval);
                    }
                }
                S.c[(hh * kRB + ro) * kKT + co] = cval;
            }
            __syncthreads();
            if (pass == 0) {
                // running max and sum of exp per (head, row): one thread each
                for (int idx = tid; idx < c_h * kRB; idx += kThreads) {
                    const float *crow = S.c + idx * kKT;
                    float mx = S.m[idx];
                    for (int co = 0; co < kKT; ++co) mx = fmaxf(mx, crow[co]);
                    if (mx == -INFINITY) continue;           // no live key yet
                    float sum = S.l[idx] * expf(S.m[idx] - mx);
                    for (int co = 0; co < kKT; ++co) sum += expf(crow[co] - mx);
                    S.m[idx] = mx;
                    S.l[idx] = sum;
                }
                __syncthreads();
                continue;
            }
            // pass 2: P in place of C, then the v rows of the tile
            for (int idx = tid; idx < c_h * kRB * kKT; idx += kThreads) {
                const int hr = idx / kKT;                        // head * kRB + row
                S.c[idx] = expf(S.c[idx] - S.m[hr]) / S.l[hr];   // exp(-inf) = 0 masks
            }
            for (int idx = tid; idx < c_h * kKT * d; idx += kThreads) {
                const int hh = idx / (kKT * d), co = (idx / d) % kKT, e = idx % d;
                const int j = j0 + co;
                S.kv[(hh * kKT + co) * d + e] = j < T ? v[((head0 + hh) * T + j) * (size_t)d + e] : 0.f;
            }
            __syncthreads();
            // O^h[ro][e] += sum_co (sum_h' w[h][h'] P^h'[ro][co]) V^h[co][e]
            for (int idx = tid; idx < kRB * c_h * d; idx += kThreads) {
                const int ro = idx / (c_h * d), ho = (idx / d) % c_h, e = idx % d;
                float acc = S.o[idx];
                for (int co = 0; co < kKT; ++co) {
                    float a = 0.f;
                    for (int hi = 0; hi < c_h; ++hi)
                        a = fmaf(S.w[ho * c_h + hi], S.c[(hi * kRB + ro) * kKT + co], a);
                    acc = fmaf(a, S.kv[(ho * kKT + co) * d + e], acc);
                }
                S.o[idx] = acc;
            }
            __syncthreads();
        }
    }
    // GroupNorm per (row, head): one warp per pair, lanes over the d channels
    const int warp = tid / 32, lane = tid % 32;
    for (int pr = warp; pr < kRB * c_h; pr += kThreads / 32) {
        const int ro = pr / c_h, ho = pr % c_h;
        const int i = i0 + ro;
        if (i >= T) continue;
        const float *orow = S.o + (ro * c_h + ho) * d;
        float s = 0.f;
        for (int e = lane; e < d; e += 32) s += orow[e];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        const float mean = s / d;
        float s2 = 0.f;
        for (int e = lane; e < d; e += 32) s2 += (orow[e] - mean) * (orow[e] - mean);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
        const float inv = 1.f / sqrtf(s2 / d + eps);
        const int h = g * c_h + ho;
        const float scale = gate ? 1.f / (1.f + expf(-gate[h])) : depth_scale;
        float *dst = out + ((size_t)b * T + i) * ((size_t)H * d) + (size_t)h * d;
        for (int e = lane; e < d; e += 32) {
            const size_t ch = (size_t)h * d + e;
            dst[e] = scale * ((orow[e] - mean) * inv * gn_weight[ch] + gn_bias[ch]);
        }
    }
}

}  // namespace

bool fused_f32_supported(const mta_shape &s)
{
    return s.io == MTA_F32 && s.c_h <= 16 && s.c_h * s.d <= kMaxCHD && s.d <= kMaxD &&
           s.c_q <= kMaxCq && s.c_k <= kMaxCk;
}

mta_status launch_fused_f32(const mta_shape &s, const ForwardArgs &a, cudaStream_t st,
                            const Trace &tr)
{
    const size_t smem = sizeof(F32Smem);
    if (cudaFuncSetAttribute(k_mta_fused_f32, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return MTA_ERR_CUDA;
    dim3 grid((s.T + kRB - 1) / kRB, s.B * (s.H / s.c_h));
    tr.before(0, st);
    k_mta_fused_f32<<<grid, kThreads, smem, st>>>(
        (const float *)a.q, (const float *)a.k, (const float *)a.v, a.w_kq, a.w_head,
        a.gn_weight, a.gn_bias, a.depth_scale, a.gate, s.gn_eps, (float *)a.out, s.T, s.H, s.d,
        s.c_q, s.c_k, s.c_h);
    tr.after(0, st);
    return cudaGetLastError() == cudaSuccess ? MTA_OK : MTA_ERR_CUDA;
}

}  // namespace mta
