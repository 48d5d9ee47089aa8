// Internal interfaces between the C-ABI layer (api.cu) and the kernel
// translation units.  Not installed; the public ABI is include/mta.h.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "mta.h"

namespace mta {

// Tensor arguments of one forward call, all device pointers.
struct ForwardArgs {
    const void *q, *k, *v;
    const float *w_kq, *w_head, *gn_weight, *gn_bias;
    float depth_scale;
    void *out;
    const float *gate = nullptr;   // [H] sigmoid-gate logits; null: depth scale
    // Steps after the first head mix (materialised path only): a key-query
    // kernel on the probabilities and a second head mix; null: left out.
    // On that path w_kq and w_head may be null too (the step is left out).
    const float *w_kq_post = nullptr, *w_head_post = nullptr;
    // Before the softmax: a mix of the logits after the w_kq conv, and the
    // exact indicator of Eq. (4) for that conv instead of Mask_0.
    const float *w_head_pre = nullptr;
    int exact_mask = 0;
    // The 3-D kernel [H/c_h][c_h][c_h][c_q][c_k] in place of w_kq, or null.
    const float *w_kq_3d = nullptr;
};

// Optional CUDA events recorded around the kernel launches of one call.
struct Trace {
    void *const *events = nullptr;
    int n = 0;
    void before(int launch, cudaStream_t st) const {
        if (2 * launch + 1 < n) cudaEventRecord((cudaEvent_t)events[2 * launch], st);
    }
    void after(int launch, cudaStream_t st) const {
        if (2 * launch + 1 < n) cudaEventRecord((cudaEvent_t)events[2 * launch + 1], st);
    }
};

inline size_t bh_tt(const mta_shape &s) {
    return (size_t)s.B * s.H * (size_t)s.T * (size_t)s.T;
}

// Materialised chain (unfused.cu).
// Launchers of its kernels, also used by the backward pass (backward.cu):
//  logits        map[bh][i][j] = q_i . k_j / sqrt(d) for j <= i + band, 0 above
//  logits_f32_io map[bh][i][j] = scale * a_i . b_j for j <= i (a fp32 [B*H][T][d],
//                b of the I/O type)
//  launch_conv   the Eq. (4) key-query convolution of src into dst (j <= i)
//  softmax_mix   softmax rows of map1 and the Eq. (7) head mix (w_head null:
//                the identity) into dst
//  head_mix      Eq. (7) without a softmax
mta_status logits(const mta_shape &s, const void *q, const void *k, float *map0, int band,
                  cudaStream_t st);
void logits_f32_io(const mta_shape &s, const float *a, const void *b, float scale, float *map,
                   cudaStream_t st);
void launch_conv(const mta_shape &s, const float *src, float *dst, const float *w_kq, int band,
                 int nin, cudaStream_t st);
mta_status softmax_mix(const mta_shape &s, const float *map1, float *dst, const float *w_head,
                       int mode, cudaStream_t st);
mta_status head_mix(const mta_shape &s, const float *src, float *dst, const float *w_head,
                    cudaStream_t st);
size_t unfused_workspace_bytes(const mta_shape &s);
constexpr int kUnfusedKernels = 4;
// Kernel names of the default chain for shape s (tensor-core logits and
// A V for bf16 I/O at d = 64 or 128, CUDA-core fp32 otherwise).
const char *unfused_kernel_name(const mta_shape &s, int index);
// Launch sequence of launch_unfused for the steps a names (at most
// kMaxChainKernels); fills names[] in launch order and returns the count.
constexpr int kMaxChainKernels = 7;
int unfused_chain(const mta_shape &s, const ForwardArgs &a, const char **names);
// Tensor-core kernels of the chain (unfused_tc.cu), bf16 I/O with d = 64 or
// 128 (chain_tc_supported): logits_tc as `logits`, pv_groupnorm_tc the
// A V + GroupNorm + output-scale step into a.out.
bool chain_tc_supported(const mta_shape &s);
mta_status logits_tc(const mta_shape &s, const void *q, const void *k, float *map0, int band,
                     cudaStream_t st);
mta_status pv_groupnorm_tc(const mta_shape &s, const float *amap, const ForwardArgs &a,
                           cudaStream_t st);
// fp32 products of the backward pass on tensor cores (3xTF32, the accuracy of
// an fp32 dot product), for d = 64 or 128 (mm_tf32_supported):
//  causal_mm_tf32  out[bh][r][:] = scale * sum over c of M[r][c] X[c][:], with
//                  trans false: M = map rows, c <= r; trans true: M = map^T,
//                  c >= r.  X is [B*H][T][d], of the I/O type when x_io, else
//                  fp32; out fp32 [B*H][T][d]
//  logits_f32_tf32 map[bh][i][j] = scale * a_i . b_j for j <= i, 0 above (a fp32
//                  [B*H][T][d], b of the I/O type)
bool mm_tf32_supported(const mta_shape &s);
mta_status causal_mm_tf32(const mta_shape &s, bool trans, const float *map, const void *x,
                          bool x_io, float *out, float scale, cudaStream_t st);
mta_status logits_f32_tf32(const mta_shape &s, const float *a, const void *b, float scale,
                           float *map, cudaStream_t st);
// Reads and clears, in one atomic step on stream `st`, the device error word
// of these kernels (bit 0: a bounded wait expired), then synchronises `st`;
// ~0u when a CUDA call failed.
unsigned int chain_take_error(cudaStream_t st);
mta_status launch_unfused(const mta_shape &s, const ForwardArgs &a, void *ws, cudaStream_t st,
                          const Trace &tr);
mta_status launch_debug_attention(const mta_shape &s, const void *q, const void *k,
                                  const float *w_kq, const float *w_head, float *attn, int stage,
                                  void *ws, cudaStream_t st);

// Backward pass (backward.cu): gradients of the default composition, on
// materialised maps in fp32.  Output pointers are device memory, fp32.
struct BackwardArgs {
    const void *dout;          // [B][T][H*d], I/O type
    float *dq, *dk, *dv;       // [B][H][T][d]
    float *dw_kq;              // [H][c_q][c_k]
    float *dw_head;            // [H/c_h][c_h][c_h]
    float *dgn_weight, *dgn_bias;   // [H*d]
    float *dgate;              // [H], with a gate only
};
constexpr int kBackwardKernels = 14;
const char *backward_kernel_name(const mta_shape &s, int index);
size_t backward_workspace_bytes(const mta_shape &s);
mta_status launch_backward(const mta_shape &s, const ForwardArgs &a, const BackwardArgs &g,
                           void *ws, cudaStream_t st, const Trace &tr);

// Fused fp32 path (fused_f32.cu): fp32 I/O, CUDA cores, no workspace.
bool fused_f32_supported(const mta_shape &s);
mta_status launch_fused_f32(const mta_shape &s, const ForwardArgs &a, cudaStream_t st,
                            const Trace &tr);

// Fused tcgen05 path (fused_tc.cu).
bool fused_supported(const mta_shape &s);
size_t fused_workspace_bytes(const mta_shape &s);
int fused_kernel_count(const mta_shape &s);
const char *fused_kernel_name(const mta_shape &s, int index);
mta_status launch_fused(const mta_shape &s, const ForwardArgs &a, void *ws, cudaStream_t st,
                        const Trace &tr);
// Device address of the static scratch mta_forward_noalloc works in (looked
// up once per device and context, with that device current).
mta_status noalloc_scratch(void **ptr);
mta_status launch_selftest_wait_timeout(long long budget_cycles, cudaStream_t st);
// Reads and clears, in one atomic step on stream `st`, the fused kernels'
// device error word of the current device (one word per device, shared by
// every stream), then synchronises `st`; ~0u when a CUDA call failed.
unsigned int fused_take_error(cudaStream_t st);

}  // namespace mta
