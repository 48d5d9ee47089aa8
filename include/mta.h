/*
 * mta.h -- C ABI of the Multi-Token Attention (MTA) forward library for
 * NVIDIA B200 (sm_100a).  Library: convolved_logit_attention_b200/libmta.so.
 *
 * What is computed (per batch entry b, head h, query i, key j, following
 * "Multi-Token Attention -- Paper Graph", section 3.4):
 *   S1  A^[i][j]  = q_i . k_j / sqrt(d)                ("Standard Multi-Head
 *                                                        Attention")
 *   S2  A0        = Mask_0(A^): zero where j > i       ("Key-Query Convolution",
 *                                                        Eq. (5), first mask)
 *   S3  C[i][j]   = sum_{i'=0}^{c_q-1} sum_{j'=-floor(c_k/2)}^{ceil(c_k/2)-1}
 *                   theta_h[i'][j'] A0[i-i'][j-j']     (Eq. (4) index ranges;
 *                   taps outside [0,T)^2 read zero)
 *   S4  C[i][j]   = -inf where j > i                   (Eq. (5), second mask)
 *   S5  P^h       = softmax over j of C                ("Standard MHA")
 *   S6  A^h_new   = sum_{h' in group(h)} w_g[h][h'] P^h'
 *                   (groups of c_h consecutive heads; "Head Mixing
 *                   Convolution", Eq. (7), applied after the softmax)
 *   S7  O^h       = A^h_new V^h
 *   S8  y         = GroupNorm over each head's d values (biased variance,
 *                   eps inside the root) with per-channel gamma, beta
 *                   ("Group Normalization with Sigmoid Gating"; one group
 *                   per head)
 *   S9  out       = depth_scale * y                    ("Article Overview:
 *                   Multi-Token Attention", section 2, "Group Normalization
 *                   with Depth Scaling")
 *
 * Conventions shared by every entry point:
 *   - Every tensor pointer is DEVICE memory owned by the caller; the library
 *     never allocates, frees or keeps a pointer after the call returns.
 *   - Tensors are dense and contiguous, row-major, with these layouts:
 *       q, k, v    [B][H][T][d]       dtype shape->io (fp32 or bf16)
 *       w_kq       [H][c_q][c_k]      fp32; tap (i', j') at [h][i'][j'+floor(c_k/2)]
 *       w_head     [H/c_h][c_h][c_h]  fp32; [group][output head][input head]
 *       gn_weight  [H*d], gn_bias [H*d]   fp32, channel h*d + e
 *       out        [B][T][H*d]        dtype shape->io (the head concatenation)
 *   - Device pointers must be 16-byte aligned; the workspace 256-byte aligned.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t passed as a
 *     plain pointer; NULL means the legacy default stream).  Argument errors
 *     are detected on the host before anything is enqueued, and nothing is
 *     enqueued when a call returns an error.
 *   - Errors are returned as mta_status codes; the library never aborts,
 *     throws or prints.  A device-side wait that runs out of its bound makes
 *     the kernel return early and raises a flag that mta_sync_status()
 *     reports as MTA_ERR_DEVICE_TIMEOUT.
 */
#ifndef MTA_H
#define MTA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Symbols of the ABI are exported; everything else in the library is hidden. */
#if defined(__GNUC__)
#define MTA_API __attribute__((visibility("default")))
#else
#define MTA_API
#endif

typedef enum {
    MTA_OK = 0,
    MTA_ERR_INVALID_ARG = -1,    /* null pointer, non-positive size, H % c_h != 0 */
    MTA_ERR_UNSUPPORTED = -2,    /* shape outside the supported ranges below */
    MTA_ERR_ALIGNMENT = -3,      /* pointer not 16-byte (workspace: 256-byte) aligned */
    MTA_ERR_WORKSPACE = -4,      /* workspace smaller than the *_workspace_size query */
    MTA_ERR_CUDA = -5,           /* a CUDA runtime call failed */
    MTA_ERR_DEVICE_TIMEOUT = -6, /* a bounded device-side wait expired */
    MTA_ERR_RANGE = -7           /* the fused path met inputs outside its accuracy domain
                                    (beyond fp16, or non-finite): see mta_forward */
} mta_status;

typedef enum { MTA_F32 = 0, MTA_BF16 = 1 } mta_dtype;

/* Problem description.  Supported ranges: B, H, T >= 1 with B*H <= 65535;
 * 8 <= d <= 128 with d % 8 == 0; 1 <= c_q <= 8; 1 <= c_k <= 15;
 * c_h in {1, 2, 4, 8, 16} with H % c_h == 0; gn_eps > 0 (1e-5 is the usual
 * GroupNorm default; the pages do not state one).  Violations of the
 * arithmetic constraints (non-positive sizes, H % c_h, gn_eps) are
 * MTA_ERR_INVALID_ARG; sizes outside the supported ranges are
 * MTA_ERR_UNSUPPORTED. */
typedef struct {
    int B, H, T, d, c_q, c_k, c_h;
    mta_dtype io;
    float gn_eps;
} mta_shape;

/* Which device path mta_forward takes for a shape. */
typedef enum {
    MTA_PATH_FUSED_TC = 0,       /* bf16 I/O, d in {64, 128}: fused tcgen05 kernels, no T x T
                                    map in HBM */
    MTA_PATH_MATERIALISED = 1,   /* the S1..S9 chain of mta_forward_unfused */
    MTA_PATH_FUSED_F32 = 2       /* fp32 I/O with c_h * d <= 256: one fused kernel on CUDA
                                    cores (fp32 arithmetic), no T x T map in HBM, no
                                    workspace */
} mta_path;

/* Library ABI version (major * 10000 + minor * 100 + patch). */
MTA_API int mta_version(void);

/* Static text for a status code; never NULL. */
MTA_API const char *mta_status_string(mta_status status);

/* The path mta_forward uses for *shape (an invalid shape reports
 * MTA_PATH_MATERIALISED; validation happens in the call itself). */
MTA_API mta_path mta_forward_path(const mta_shape *shape);

/* Bytes of device workspace mta_forward needs for *shape (0 on an invalid
 * shape).  Sized for the path mta_forward_path() names. */
MTA_API size_t mta_workspace_size(const mta_shape *shape);

/* Bytes of device workspace mta_forward_unfused and mta_debug_attention need:
 * two fp32 [B][H][T][T] maps. */
MTA_API size_t mta_unfused_workspace_size(const mta_shape *shape);

/* The MTA forward S1..S9 above, out = depth_scale * GN(...), written to out.
 * The fused path computes the folded logits on tensor cores with fp16
 * operands (q and the folded keys) and P V with bf16 operands, both with fp32
 * accumulation.  The materialised path keeps fp32 maps; for bf16 I/O at
 * d = 64 or 128 its Q K^T runs on tensor cores from the bf16 inputs (exact
 * products, fp32 accumulation) and its A V with the attention weights rounded
 * to bf16, otherwise both are fp32 CUDA-core products.  The fused path
 * subtracts, on the tiles next to the diagonal, the future terms that Mask_0
 * removes; those terms were computed with fp16 operands, so the logits there
 * carry an absolute error of about 2^-11 |theta| |q| |k| / sqrt(d) per future
 * term (negligible for activations of order 10, ruinous for order 1e4).  A
 * 128-row block of queries or of folded keys beyond the fp16 range is scaled
 * by a power of two before the rounding and its logits scaled back exactly,
 * so the output stays finite, and the call's next mta_sync_status() reports
 * MTA_ERR_RANGE: such inputs are outside the fused path's accuracy domain and
 * mta_forward_unfused (fp32 logits, and bf16 operands, which have the fp32
 * exponent range) is the path for them.  A non-finite
 * q, k or v, or anything that makes an output non-finite, is reported the
 * same way.
 * The workspace is scratch owned by the caller for the duration of the
 * enqueued work; its contents on entry are ignored. */
MTA_API mta_status mta_forward(const mta_shape *shape, const void *q, const void *k, const void *v,
                       const float *w_kq, const float *w_head, const float *gn_weight,
                       const float *gn_bias, float depth_scale, void *out,
                       void *workspace, size_t workspace_bytes, void *stream);

/* The forward with the pages' default output scale ("Multi-Token Attention
 * -- Paper Graph", "Group Normalization with Sigmoid Gating"): head h of the
 * GroupNorm output (after its affine) is multiplied by sigmoid(gate[h]),
 * out = GN(...) * sigmoid(g), in place of a depth scale.  gate is a caller-
 * owned device array of H floats (4-byte aligned); NULL is MTA_ERR_INVALID_ARG.
 * Path, workspace and every other argument as for mta_forward. */
MTA_API mta_status mta_forward_gated(const mta_shape *shape, const void *q, const void *k,
                             const void *v, const float *w_kq, const float *w_head,
                             const float *gn_weight, const float *gn_bias, const float *gate,
                             void *out, void *workspace, size_t workspace_bytes, void *stream);

/* The same forward computed step by step with the T x T maps materialised in
 * the workspace (S1+S2 logits, S3+S4 conv, S5+S6 softmax and mix, S7..S9
 * PV with the GroupNorm epilogue), all arithmetic in fp32.  Same arguments
 * and contract as mta_forward. */
MTA_API mta_status mta_forward_unfused(const mta_shape *shape, const void *q, const void *k,
                               const void *v, const float *w_kq, const float *w_head,
                               const float *gn_weight, const float *gn_bias, float depth_scale,
                               void *out, void *workspace, size_t workspace_bytes,
                               void *stream);

/* Debug view of the attention maps for small problems (T <= 2048):
 * attn [B][H][T][T] fp32 receives the pre-mix softmax P (stage 0) or the
 * post-mix A_new (stage 1), with zeros above the diagonal.  Workspace as for
 * mta_forward_unfused.  Any other stage is MTA_ERR_INVALID_ARG; T > 2048 is
 * MTA_ERR_UNSUPPORTED. */
MTA_API mta_status mta_debug_attention(const mta_shape *shape, const void *q, const void *k,
                               const float *w_kq, const float *w_head, float *attn, int stage,
                               void *workspace, size_t workspace_bytes, void *stream);

/* Kernel launches one mta_forward (unfused == 0) or mta_forward_unfused
 * (unfused != 0) call makes for *shape, and the name of launch `index`
 * (NULL when out of range or the shape is invalid).  For tracing. */
MTA_API int mta_kernel_count(const mta_shape *shape, int unfused);
MTA_API const char *mta_kernel_name(const mta_shape *shape, int unfused, int index);

/* mta_forward (unfused == 0) or mta_forward_unfused (unfused != 0) that also
 * records caller-created CUDA events (cudaEvent_t handles passed as plain
 * pointers) on `stream` around its kernel launches: events[2*i] just before
 * and events[2*i+1] just after launch i, for i < n_events / 2.  The events
 * stay owned by the caller.  Same contract as the untraced call otherwise;
 * a NULL `events` with n_events == 0 records nothing. */
MTA_API mta_status mta_forward_traced(int unfused, const mta_shape *shape, const void *q,
                                      const void *k, const void *v, const float *w_kq,
                                      const float *w_head, const float *gn_weight,
                                      const float *gn_bias, float depth_scale, void *out,
                                      void *workspace, size_t workspace_bytes, void *stream,
                                      void *const *events, int n_events);

/* Diagnostic for the timeout path: enqueues one single-thread kernel that
 * waits on a shared-memory barrier nothing ever completes, with the same
 * bounded wait the fused kernels use, cut off after `budget_cycles` SM clock
 * cycles (must be in (0, 2^31)).  The kernel then raises the device error
 * flag and returns, so the next mta_sync_status() reports
 * MTA_ERR_DEVICE_TIMEOUT (and clears the flag) while the CUDA context stays
 * usable. */
MTA_API mta_status mta_selftest_wait_timeout(long long budget_cycles, void *stream);

/* Bytes of the static device scratch mta_forward_noalloc works in. */
#define MTA_NOALLOC_SCRATCH_BYTES (32u << 20)

/* mta_forward for callers that cannot allocate device memory.  The pages
 * have no counterpart: this is a convenience of the interface, not of the
 * method.  Some callers are handed only their input and output buffers and
 * have no way to obtain scratch, for example a plugin whose host framework
 * owns every device allocation, or an application that reserves all of its
 * device memory up front and forbids allocations afterwards.  This entry
 * takes the same arguments as mta_forward minus the workspace and runs the
 * same fused kernels in a scratch area that lives inside the library: a
 * MTA_NOALLOC_SCRATCH_BYTES (32 MiB) device array that every GPU which loads
 * the library keeps until the process exits.  It allocates nothing and frees
 * nothing.
 *   - Shapes whose fused-path scratch (mta_workspace_size) exceeds
 *     MTA_NOALLOC_SCRATCH_BYTES return MTA_ERR_WORKSPACE; shapes that do not
 *     take the fused path (mta_forward_path) return MTA_ERR_UNSUPPORTED.
 *     Nothing is enqueued in either case.
 *   - The first call on a device looks up the scratch's device address (with
 *     that device current); make that first call before any stream capture.
 *     The address is kept per device and context: after the device's context
 *     is destroyed (cudaDeviceReset) the next call looks it up again, so make
 *     that call outside stream capture as well.
 *   - All calls on a device share the one scratch area and leave their data
 *     in it.  Every byte a call reads there it has written first, so stale
 *     contents do no harm, but calls whose work overlaps on the GPU (other
 *     streams, other host threads) race on it: serialise them. */
MTA_API mta_status mta_forward_noalloc(const mta_shape *shape, const void *q, const void *k,
                                       const void *v, const float *w_kq, const float *w_head,
                                       const float *gn_weight, const float *gn_bias,
                                       float depth_scale, void *out, void *stream);

/* One composition of the module ("Multi-Token Attention -- Paper Graph",
 * "Putting Everything Together: The Full MTA Module").  The steps run in
 * this fixed order, each bracketed one only when its weights are given:
 *   S1+S2, [S3 with w_kq], [L1: head mix of the logits with w_head_pre],
 *   S4, S5, [S6 with w_head],
 *   [P1: conv of the probabilities with w_kq_post, zero where j > i],
 *   [P2: Eq. (7) head mix with w_head_post], S7..S9
 * P1 is the post-softmax variant of "Key-Query Convolution":
 * A1 -> Mask_0(Conv2d_theta(A1)), with the index ranges and zero padding of
 * S3.  L1 is the pre-softmax version of "Head Mixing Convolution": the
 * logits of a group's heads are mixed, on the keys j <= i, before S4; S3
 * then L1 is the separable case of the 3-D convolution of "Putting
 * Everything Together" ("both pre-softmax").  exact_mask != 0 replaces S2's
 * Mask_0 for S3 by the indicator of Eq. (4): the tap (i', j') of output
 * (i, j) adds theta q_{i-i'} k_{j-j'} / sqrt(d) whenever key j - j' <= i
 * (Mask_0 keeps it only for j - j' <= i - i').  The pages' default is
 * {w_kq, w_head}; the repeated MTA convolution ("repeat this operation") is
 * {w_kq, w_head, w_kq_post, w_head_post}; "both post-softmax" is
 * {w_kq_post, w_head_post}.  Both key-query kernels are [H][c_q][c_k] and the
 * three head mixes [H/c_h][c_h][c_h], laid out as w_kq and w_head above;
 * pointers are device memory, 16-byte aligned, NULL for a step left out.
 * w_kq_3d [H/c_h][c_h][c_h][c_q][c_k] is the general 3-D kernel of "Both
 * pre-softmax (3D convolution view)": S3 becomes C^h = sum over the input
 * heads h' of h's group of the 2-D conv of A0^{h'} with
 * w_kq_3d[group][h][h'] (tap layout as w_kq), under either masking.  Giving
 * both w_kq and w_kq_3d is MTA_ERR_INVALID_ARG. */
typedef struct {
    const float *w_kq;         /* S3 before the softmax, or NULL */
    const float *w_head;       /* S6 right after the softmax, or NULL */
    const float *w_kq_post;    /* P1 on the probabilities, or NULL */
    const float *w_head_post;  /* P2 after P1, or NULL */
    const float *w_head_pre;   /* L1 on the logits, or NULL */
    int exact_mask;            /* nonzero: S3 under Eq. (4)'s indicator */
    const float *w_kq_3d;      /* the 3-D kernel in place of w_kq, or NULL (below) */
} mta_composition;

/* Bytes of device workspace mta_forward_composed needs (0 on an invalid
 * shape or a NULL composition): mta_workspace_size() for the default
 * composition (either masking), two fp32 [B][H][T][T] maps for every other
 * one. */
MTA_API size_t mta_composed_workspace_size(const mta_shape *shape, const mta_composition *comp);

/* The forward of the composition *comp, written to out.  The default
 * composition {w_kq, w_head} takes mta_forward's path (fused where
 * mta_forward_path says so), under either masking: with exact_mask the fused
 * kernels change only which taps the Mask_0 correction table subtracts
 * (those whose key lies past the output's query instead of past the tap's
 * own query).  Every other composition runs on the materialised chain, in
 * fp32, with P1 as a second conv launch and P2 as a mix-only launch.  gate is NULL for
 * out = depth_scale * GN(...), or a device array of H floats (4-byte
 * aligned) for the sigmoid gate of mta_forward_gated, depth_scale then
 * ignored.  A NULL comp is MTA_ERR_INVALID_ARG; every other argument and the
 * contract are as for mta_forward. */
MTA_API mta_status mta_forward_composed(const mta_shape *shape, const void *q, const void *k,
                                        const void *v, const mta_composition *comp,
                                        const float *gn_weight, const float *gn_bias,
                                        float depth_scale, const float *gate, void *out,
                                        void *workspace, size_t workspace_bytes, void *stream);

/* mta_forward_composed that records events around its launches, as
 * mta_forward_traced does; the launches are those mta_composed_kernel_name
 * lists, in order. */
MTA_API mta_status mta_forward_composed_traced(const mta_shape *shape, const void *q,
                                               const void *k, const void *v,
                                               const mta_composition *comp,
                                               const float *gn_weight, const float *gn_bias,
                                               float depth_scale, const float *gate, void *out,
                                               void *workspace, size_t workspace_bytes,
                                               void *stream, void *const *events, int n_events);

/* Kernel launches of one mta_forward_composed call and the name of launch
 * `index` (0 / NULL for an invalid shape, a NULL comp or an index out of
 * range). */
MTA_API int mta_composed_kernel_count(const mta_shape *shape, const mta_composition *comp);
MTA_API const char *mta_composed_kernel_name(const mta_shape *shape, const mta_composition *comp,
                                             int index);

/* Backward pass ("Multi-Token Attention -- Paper Graph", section 3.4, the
 * forward S1..S9 above; the pages report training cost, Table 9, but give no
 * gradients, so these are the forward's own by the chain rule).  Given
 * dout = dL/d(out) [B][T][H*d] (dtype shape->io), writes the gradient of L
 * with respect to every input, all fp32, caller-owned device memory:
 *   dq, dk, dv           [B][H][T][d]
 *   dw_kq                [H][c_q][c_k]       (layout of w_kq)
 *   dw_head              [H/c_h][c_h][c_h]   (layout of w_head)
 *   dgn_weight, dgn_bias [H*d]
 *   dgate                [H], only with gate != NULL (out = GN(...) * sigmoid(g),
 *                        as mta_forward_gated; depth_scale is then ignored);
 *                        NULL exactly when gate is NULL, else MTA_ERR_INVALID_ARG.
 * Every output is overwritten (not accumulated into).  The forward maps are
 * recomputed in the workspace (mta_backward_workspace_size: three fp32
 * [B][H][T][T] maps plus O and partial sums), and every step runs in fp32 on
 * the materialised chain; the parameter gradients are sums of per-block
 * partials in a fixed order, so repeated calls give identical bits.  Pointers
 * 16-byte aligned (gate and dgate 4-byte), the workspace 256-byte aligned;
 * argument errors as for mta_forward, nothing enqueued on an error. */
MTA_API size_t mta_backward_workspace_size(const mta_shape *shape);
MTA_API mta_status mta_backward(const mta_shape *shape, const void *q, const void *k,
                                const void *v, const float *w_kq, const float *w_head,
                                const float *gn_weight, const float *gn_bias, float depth_scale,
                                const float *gate, const void *dout, float *dq, float *dk,
                                float *dv, float *dw_kq, float *dw_head, float *dgn_weight,
                                float *dgn_bias, float *dgate, void *workspace,
                                size_t workspace_bytes, void *stream);

/* mta_backward that records caller-created events around its launches, as
 * mta_forward_traced does; the launches are those mta_backward_kernel_name
 * lists (the last entry covers the final reductions). */
MTA_API mta_status mta_backward_traced(const mta_shape *shape, const void *q, const void *k,
                                       const void *v, const float *w_kq, const float *w_head,
                                       const float *gn_weight, const float *gn_bias,
                                       float depth_scale, const float *gate, const void *dout,
                                       float *dq, float *dk, float *dv, float *dw_kq,
                                       float *dw_head, float *dgn_weight, float *dgn_bias,
                                       float *dgate, void *workspace, size_t workspace_bytes,
                                       void *stream, void *const *events, int n_events);
MTA_API int mta_backward_kernel_count(const mta_shape *shape);
MTA_API const char *mta_backward_kernel_name(const mta_shape *shape, int index);

/* Synchronises `stream`, then reports (and clears) the device error flags:
 * MTA_ERR_DEVICE_TIMEOUT if a kernel's bounded wait expired, MTA_ERR_RANGE if
 * the fused path met inputs beyond fp16 or non-finite ones, MTA_ERR_CUDA if the
 * synchronisation itself failed, MTA_OK otherwise.  The flags are two words
 * per device (one for the fused kernels, one for the materialised chain's
 * tensor-core kernels), shared by every stream and caller of the library on
 * that device: each word is read and cleared in one atomic step (a small
 * kernel on `stream`), so no raised flag is lost, but a call reports flags
 * raised by any work on the device since the previous report. */
MTA_API mta_status mta_sync_status(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MTA_H */
