// C-ABI entry points of libmta.so (declared in include/mta.h): argument
// validation on the host, workspace queries, and dispatch to the kernels.
// Nothing is enqueued unless every check passes.
#include <cuda_runtime.h>
#include <stdint.h>

#include "mta.h"
#include "mta_internal.h"

namespace {

bool aligned(const void *p, uintptr_t a) { return ((uintptr_t)p % a) == 0; }

bool is_pow2_ch(int c) { return c == 1 || c == 2 || c == 4 || c == 8 || c == 16; }

mta_status check_shape(const mta_shape *s)
{
    if (!s) return MTA_ERR_INVALID_ARG;
    if (s->B < 1 || s->H < 1 || s->T < 1 || s->d < 1 || s->c_q < 1 || s->c_k < 1 || s->c_h < 1)
        return MTA_ERR_INVALID_ARG;
    if (s->H % s->c_h != 0) return MTA_ERR_INVALID_ARG;
    if (!(s->gn_eps > 0.f)) return MTA_ERR_INVALID_ARG;
    if (s->io != MTA_F32 && s->io != MTA_BF16) return MTA_ERR_INVALID_ARG;
    if (s->d < 8 || s->d > 128 || s->d % 8 != 0) return MTA_ERR_UNSUPPORTED;
    if (s->c_q > 8 || s->c_k > 15 || !is_pow2_ch(s->c_h)) return MTA_ERR_UNSUPPORTED;
    // grid dimensions of the materialised kernels and 32-bit row counts
    if ((long long)s->B * s->H > 65535 || s->T > 65535 * 32) return MTA_ERR_UNSUPPORTED;
    return MTA_OK;
}

mta_status check_tensors(const void *q, const void *k, const void *v, const float *w_kq,
                         const float *w_head, const float *gn_weight, const float *gn_bias,
                         const void *out)
{
    const void *ptrs[] = {q, k, v, w_kq, w_head, gn_weight, gn_bias, out};
    for (const void *p : ptrs)
        if (!p) return MTA_ERR_INVALID_ARG;
    for (const void *p : ptrs)
        if (!aligned(p, 16)) return MTA_ERR_ALIGNMENT;
    return MTA_OK;
}

mta_status check_workspace(const void *ws, size_t have, size_t need)
{
    if (need == 0) return MTA_OK;
    if (!ws) return MTA_ERR_INVALID_ARG;
    if (!aligned(ws, 256)) return MTA_ERR_ALIGNMENT;
    if (have < need) return MTA_ERR_WORKSPACE;
    return MTA_OK;
}

}  // namespace

extern "C" {

int mta_version(void) { return 100; }

const char *mta_status_string(mta_status st)
{
    switch (st) {
        case MTA_OK: return "ok";
        case MTA_ERR_INVALID_ARG: return "invalid argument";
        case MTA_ERR_UNSUPPORTED: return "unsupported shape";
        case MTA_ERR_ALIGNMENT: return "misaligned pointer";
        case MTA_ERR_WORKSPACE: return "workspace too small";
        case MTA_ERR_CUDA: return "CUDA runtime error";
        case MTA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
        case MTA_ERR_RANGE: return "input outside the fused path's accuracy domain (beyond fp16 or non-finite)";
    }
    return "unknown status";
}

namespace {

// The path of a forward call: the fused kernels for the shapes they take
// (the fp32 one has no exact-mask variant), else the materialised chain.
mta_path path_of(const mta_shape &s, int unfused, int exact)
{
    if (unfused) return MTA_PATH_MATERIALISED;
    if (mta::fused_supported(s)) return MTA_PATH_FUSED_TC;
    if (!exact && mta::fused_f32_supported(s)) return MTA_PATH_FUSED_F32;
    return MTA_PATH_MATERIALISED;
}

size_t path_workspace(const mta_shape &s, mta_path p)
{
    switch (p) {
        case MTA_PATH_FUSED_TC: return mta::fused_workspace_bytes(s);
        case MTA_PATH_FUSED_F32: return 0;
        default: return mta::unfused_workspace_bytes(s);
    }
}

}  // namespace

mta_path mta_forward_path(const mta_shape *s)
{
    if (check_shape(s) != MTA_OK) return MTA_PATH_MATERIALISED;
    return path_of(*s, 0, 0);
}

size_t mta_workspace_size(const mta_shape *s)
{
    if (check_shape(s) != MTA_OK) return 0;
    return path_workspace(*s, path_of(*s, 0, 0));
}

size_t mta_unfused_workspace_size(const mta_shape *s)
{
    if (check_shape(s) != MTA_OK) return 0;
    return mta::unfused_workspace_bytes(*s);
}

namespace {

mta_status forward_impl(int unfused, const mta_shape *s, const void *q, const void *k,
                        const void *v, const float *w_kq, const float *w_head,
                        const float *gn_weight, const float *gn_bias, float depth_scale,
                        const float *gate, void *out, void *workspace, size_t workspace_bytes,
                        void *stream, void *const *events, int n_events, int exact_mask = 0)
{
    mta_status rc = check_shape(s);
    if (rc == MTA_OK) rc = check_tensors(q, k, v, w_kq, w_head, gn_weight, gn_bias, out);
    if (rc != MTA_OK) return rc;
    if (n_events < 0 || (n_events > 0 && !events)) return MTA_ERR_INVALID_ARG;
    const mta_path path = path_of(*s, unfused, exact_mask);
    rc = check_workspace(workspace, workspace_bytes, path_workspace(*s, path));
    if (rc != MTA_OK) return rc;
    mta::ForwardArgs a{q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, out, gate};
    a.exact_mask = exact_mask;
    mta::Trace tr;
    tr.events = events;
    tr.n = n_events;
    cudaStream_t st = (cudaStream_t)stream;
    switch (path) {
        case MTA_PATH_FUSED_TC: return mta::launch_fused(*s, a, workspace, st, tr);
        case MTA_PATH_FUSED_F32: return mta::launch_fused_f32(*s, a, st, tr);
        default: return mta::launch_unfused(*s, a, workspace, st, tr);
    }
}

}  // namespace

mta_status mta_forward_traced(int unfused, const mta_shape *s, const void *q, const void *k,
                              const void *v, const float *w_kq, const float *w_head,
                              const float *gn_weight, const float *gn_bias, float depth_scale,
                              void *out, void *workspace, size_t workspace_bytes, void *stream,
                              void *const *events, int n_events)
{
    return forward_impl(unfused, s, q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale,
                        nullptr, out, workspace, workspace_bytes, stream, events, n_events);
}

mta_status mta_forward_gated(const mta_shape *s, const void *q, const void *k, const void *v,
                             const float *w_kq, const float *w_head, const float *gn_weight,
                             const float *gn_bias, const float *gate, void *out, void *workspace,
                             size_t workspace_bytes, void *stream)
{
    if (!gate) return MTA_ERR_INVALID_ARG;
    if (((uintptr_t)gate & 3u) != 0) return MTA_ERR_ALIGNMENT;
    return forward_impl(0, s, q, k, v, w_kq, w_head, gn_weight, gn_bias, 0.f, gate, out,
                        workspace, workspace_bytes, stream, nullptr, 0);
}

namespace {

// The pages' default composition {w_kq, w_head}, under either masking of the
// first convolution: mta_forward's path (fused where mta_forward_path says so).
bool is_default_composition(const mta_composition *c)
{
    return c->w_kq && c->w_head && !c->w_kq_post && !c->w_head_post && !c->w_head_pre &&
           !c->w_kq_3d;
}

mta_status composed_impl(const mta_shape *s, const void *q, const void *k, const void *v,
                         const mta_composition *c, const float *gn_weight, const float *gn_bias,
                         float depth_scale, const float *gate, void *out, void *workspace,
                         size_t workspace_bytes, void *stream, void *const *events, int n_events)
{
    if (!c || (c->w_kq && c->w_kq_3d)) return MTA_ERR_INVALID_ARG;
    if (gate && ((uintptr_t)gate & 3u) != 0) return MTA_ERR_ALIGNMENT;
    if (is_default_composition(c))
        return forward_impl(0, s, q, k, v, c->w_kq, c->w_head, gn_weight, gn_bias, depth_scale,
                            gate, out, workspace, workspace_bytes, stream, events, n_events,
                            c->exact_mask != 0);
    mta_status rc = check_shape(s);
    if (rc != MTA_OK) return rc;
    const void *need[] = {q, k, v, gn_weight, gn_bias, out};
    for (const void *p : need)
        if (!p) return MTA_ERR_INVALID_ARG;
    for (const void *p : need)
        if (!aligned(p, 16)) return MTA_ERR_ALIGNMENT;
    const void *opt[] = {c->w_kq, c->w_head, c->w_kq_post, c->w_head_post, c->w_head_pre,
                         c->w_kq_3d};
    for (const void *p : opt)
        if (p && !aligned(p, 16)) return MTA_ERR_ALIGNMENT;
    if (n_events < 0 || (n_events > 0 && !events)) return MTA_ERR_INVALID_ARG;
    rc = check_workspace(workspace, workspace_bytes, mta::unfused_workspace_bytes(*s));
    if (rc != MTA_OK) return rc;
    mta::ForwardArgs a{q, k, v, c->w_kq, c->w_head, gn_weight, gn_bias, depth_scale, out, gate,
                       c->w_kq_post, c->w_head_post, c->w_head_pre, c->exact_mask != 0,
                       c->w_kq_3d};
    mta::Trace tr;
    tr.events = events;
    tr.n = n_events;
    return mta::launch_unfused(*s, a, workspace, (cudaStream_t)stream, tr);
}

mta::ForwardArgs chain_args(const mta_composition *c)
{
    mta::ForwardArgs a{};
    a.w_kq = c->w_kq;
    a.w_head = c->w_head;
    a.w_kq_post = c->w_kq_post;
    a.w_head_post = c->w_head_post;
    a.w_head_pre = c->w_head_pre;
    a.exact_mask = c->exact_mask != 0;
    a.w_kq_3d = c->w_kq_3d;
    return a;
}

}  // namespace

size_t mta_composed_workspace_size(const mta_shape *s, const mta_composition *c)
{
    if (!c || check_shape(s) != MTA_OK) return 0;
    return is_default_composition(c) ? path_workspace(*s, path_of(*s, 0, c->exact_mask))
                                     : mta::unfused_workspace_bytes(*s);
}

mta_status mta_forward_composed(const mta_shape *s, const void *q, const void *k, const void *v,
                                const mta_composition *c, const float *gn_weight,
                                const float *gn_bias, float depth_scale, const float *gate,
                                void *out, void *workspace, size_t workspace_bytes, void *stream)
{
    return composed_impl(s, q, k, v, c, gn_weight, gn_bias, depth_scale, gate, out, workspace,
                         workspace_bytes, stream, nullptr, 0);
}

mta_status mta_forward_composed_traced(const mta_shape *s, const void *q, const void *k,
                                       const void *v, const mta_composition *c,
                                       const float *gn_weight, const float *gn_bias,
                                       float depth_scale, const float *gate, void *out,
                                       void *workspace, size_t workspace_bytes, void *stream,
                                       void *const *events, int n_events)
{
    return composed_impl(s, q, k, v, c, gn_weight, gn_bias, depth_scale, gate, out, workspace,
                         workspace_bytes, stream, events, n_events);
}

int mta_composed_kernel_count(const mta_shape *s, const mta_composition *c)
{
    if (!c || check_shape(s) != MTA_OK) return 0;
    if (is_default_composition(c) && !c->exact_mask) return mta_kernel_count(s, 0);
    if (is_default_composition(c) && path_of(*s, 0, 1) == MTA_PATH_FUSED_TC)
        return mta::fused_kernel_count(*s);
    const char *names[mta::kMaxChainKernels];
    return mta::unfused_chain(*s, chain_args(c), names);
}

const char *mta_composed_kernel_name(const mta_shape *s, const mta_composition *c, int index)
{
    if (!c || check_shape(s) != MTA_OK || index < 0) return nullptr;
    if (is_default_composition(c) && !c->exact_mask) return mta_kernel_name(s, 0, index);
    if (is_default_composition(c) && path_of(*s, 0, 1) == MTA_PATH_FUSED_TC)
        return mta::fused_kernel_name(*s, index);
    const char *names[mta::kMaxChainKernels];
    const int n = mta::unfused_chain(*s, chain_args(c), names);
    return index < n ? names[index] : nullptr;
}

mta_status mta_forward(const mta_shape *s, const void *q, const void *k, const void *v,
                       const float *w_kq, const float *w_head, const float *gn_weight,
                       const float *gn_bias, float depth_scale, void *out, void *workspace,
                       size_t workspace_bytes, void *stream)
{
    return mta_forward_traced(0, s, q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, out,
                              workspace, workspace_bytes, stream, nullptr, 0);
}

mta_status mta_forward_unfused(const mta_shape *s, const void *q, const void *k, const void *v,
                               const float *w_kq, const float *w_head, const float *gn_weight,
                               const float *gn_bias, float depth_scale, void *out,
                               void *workspace, size_t workspace_bytes, void *stream)
{
    return mta_forward_traced(1, s, q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, out,
                              workspace, workspace_bytes, stream, nullptr, 0);
}

mta_status mta_forward_noalloc(const mta_shape *s, const void *q, const void *k, const void *v,
                               const float *w_kq, const float *w_head, const float *gn_weight,
                               const float *gn_bias, float depth_scale, void *out, void *stream)
{
    mta_status rc = check_shape(s);
    if (rc == MTA_OK) rc = check_tensors(q, k, v, w_kq, w_head, gn_weight, gn_bias, out);
    if (rc != MTA_OK) return rc;
    if (!mta::fused_supported(*s)) return MTA_ERR_UNSUPPORTED;
    if (mta::fused_workspace_bytes(*s) > (size_t)MTA_NOALLOC_SCRATCH_BYTES) return MTA_ERR_WORKSPACE;
    void *scratch = nullptr;
    rc = mta::noalloc_scratch(&scratch);
    if (rc != MTA_OK) return rc;
    mta::ForwardArgs a{q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, out};
    const mta::Trace none;
    return mta::launch_fused(*s, a, scratch, (cudaStream_t)stream, none);
}

int mta_kernel_count(const mta_shape *s, int unfused)
{
    if (check_shape(s) != MTA_OK) return 0;
    switch (path_of(*s, unfused, 0)) {
        case MTA_PATH_FUSED_TC: return mta::fused_kernel_count(*s);
        case MTA_PATH_FUSED_F32: return 1;
        default: return mta::kUnfusedKernels;
    }
}

const char *mta_kernel_name(const mta_shape *s, int unfused, int index)
{
    if (check_shape(s) != MTA_OK || index < 0 || index >= mta_kernel_count(s, unfused))
        return nullptr;
    switch (path_of(*s, unfused, 0)) {
        case MTA_PATH_FUSED_TC: return mta::fused_kernel_name(*s, index);
        case MTA_PATH_FUSED_F32: return "k_mta_fused_f32";
        default: return mta::unfused_kernel_name(*s, index);
    }
}

mta_status mta_debug_attention(const mta_shape *s, const void *q, const void *k,
                               const float *w_kq, const float *w_head, float *attn, int stage,
                               void *workspace, size_t workspace_bytes, void *stream)
{
    mta_status rc = check_shape(s);
    if (rc != MTA_OK) return rc;
    if (stage != 0 && stage != 1) return MTA_ERR_INVALID_ARG;
    if (s->T > 2048) return MTA_ERR_UNSUPPORTED;
    const void *ptrs[] = {q, k, w_kq, w_head, attn};
    for (const void *p : ptrs)
        if (!p) return MTA_ERR_INVALID_ARG;
    for (const void *p : ptrs)
        if (!aligned(p, 16)) return MTA_ERR_ALIGNMENT;
    rc = check_workspace(workspace, workspace_bytes, mta::unfused_workspace_bytes(*s));
    if (rc != MTA_OK) return rc;
    return mta::launch_debug_attention(*s, q, k, w_kq, w_head, attn, stage, workspace,
                                       (cudaStream_t)stream);
}

size_t mta_backward_workspace_size(const mta_shape *s)
{
    if (check_shape(s) != MTA_OK) return 0;
    return mta::backward_workspace_bytes(*s);
}

int mta_backward_kernel_count(const mta_shape *s)
{
    return check_shape(s) == MTA_OK ? mta::kBackwardKernels : 0;
}

const char *mta_backward_kernel_name(const mta_shape *s, int index)
{
    if (check_shape(s) != MTA_OK || index < 0 || index >= mta::kBackwardKernels) return nullptr;
    return mta::backward_kernel_name(*s, index);
}

mta_status mta_backward_traced(const mta_shape *s, const void *q, const void *k, const void *v,
                               const float *w_kq, const float *w_head, const float *gn_weight,
                               const float *gn_bias, float depth_scale, const float *gate,
                               const void *dout, float *dq, float *dk, float *dv, float *dw_kq,
                               float *dw_head, float *dgn_weight, float *dgn_bias, float *dgate,
                               void *workspace, size_t workspace_bytes, void *stream,
                               void *const *events, int n_events)
{
    mta_status rc = check_shape(s);
    if (rc == MTA_OK) rc = check_tensors(q, k, v, w_kq, w_head, gn_weight, gn_bias, dout);
    if (rc != MTA_OK) return rc;
    const void *grads[] = {dq, dk, dv, dw_kq, dw_head, dgn_weight, dgn_bias};
    for (const void *p : grads)
        if (!p) return MTA_ERR_INVALID_ARG;
    for (const void *p : grads)
        if (!aligned(p, 16)) return MTA_ERR_ALIGNMENT;
    if ((gate == nullptr) != (dgate == nullptr)) return MTA_ERR_INVALID_ARG;
    if (gate && (!aligned(gate, 4) || !aligned(dgate, 4))) return MTA_ERR_ALIGNMENT;
    if (n_events < 0 || (n_events > 0 && !events)) return MTA_ERR_INVALID_ARG;
    rc = check_workspace(workspace, workspace_bytes, mta::backward_workspace_bytes(*s));
    if (rc != MTA_OK) return rc;
    mta::ForwardArgs a{q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, nullptr, gate};
    mta::BackwardArgs g{dout, dq, dk, dv, dw_kq, dw_head, dgn_weight, dgn_bias, dgate};
    mta::Trace tr;
    tr.events = events;
    tr.n = n_events;
    return mta::launch_backward(*s, a, g, workspace, (cudaStream_t)stream, tr);
}

mta_status mta_backward(const mta_shape *s, const void *q, const void *k, const void *v,
                        const float *w_kq, const float *w_head, const float *gn_weight,
                        const float *gn_bias, float depth_scale, const float *gate,
                        const void *dout, float *dq, float *dk, float *dv, float *dw_kq,
                        float *dw_head, float *dgn_weight, float *dgn_bias, float *dgate,
                        void *workspace, size_t workspace_bytes, void *stream)
{
    return mta_backward_traced(s, q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, gate,
                               dout, dq, dk, dv, dw_kq, dw_head, dgn_weight, dgn_bias, dgate,
                               workspace, workspace_bytes, stream, nullptr, 0);
}

mta_status mta_selftest_wait_timeout(long long budget_cycles, void *stream)
{
    if (budget_cycles <= 0 || budget_cycles >= (1ll << 31)) return MTA_ERR_INVALID_ARG;
    return mta::launch_selftest_wait_timeout(budget_cycles, (cudaStream_t)stream);
}

mta_status mta_sync_status(void *stream)
{
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MTA_ERR_CUDA;
    const unsigned int fused = mta::fused_take_error((cudaStream_t)stream);
    const unsigned int chain = mta::chain_take_error((cudaStream_t)stream);
    if (fused == ~0u || chain == ~0u) return MTA_ERR_CUDA;
    const unsigned int err = fused | chain;
    if (err & 1u) return MTA_ERR_DEVICE_TIMEOUT;
    if (err & 2u) return MTA_ERR_RANGE;
    return MTA_OK;
}

}  // extern "C"
