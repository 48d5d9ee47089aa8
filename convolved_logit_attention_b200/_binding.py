"""ctypes binding of libmta.so (the C ABI declared in include/mta.h).

Argument marshalling only: shapes, dtypes, devices and contiguity are checked,
missing outputs and workspaces are allocated through torch (device memory is
torch's job here), and the call goes to the library on the caller's current
CUDA stream.  Every step of the computation runs in the library's kernels;
there is no other implementation behind these functions, and a missing or
unloadable library raises instead of falling back.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmta.so")

MTA_F32, MTA_BF16 = 0, 1
MTA_PATH_FUSED_TC, MTA_PATH_MATERIALISED, MTA_PATH_FUSED_F32 = 0, 1, 2
STATUS = {0: "MTA_OK", -1: "MTA_ERR_INVALID_ARG", -2: "MTA_ERR_UNSUPPORTED",
          -3: "MTA_ERR_ALIGNMENT", -4: "MTA_ERR_WORKSPACE", -5: "MTA_ERR_CUDA",
          -6: "MTA_ERR_DEVICE_TIMEOUT", -7: "MTA_ERR_RANGE"}

# Every function include/mta.h declares.
EXPORTS = ("mta_version", "mta_status_string", "mta_forward_path", "mta_workspace_size",
           "mta_unfused_workspace_size", "mta_forward", "mta_forward_unfused",
           "mta_debug_attention", "mta_kernel_count", "mta_kernel_name", "mta_forward_traced",
           "mta_selftest_wait_timeout", "mta_forward_noalloc", "mta_sync_status",
           "mta_forward_gated", "mta_composed_workspace_size", "mta_forward_composed",
           "mta_forward_composed_traced", "mta_composed_kernel_count", "mta_composed_kernel_name",
           "mta_backward", "mta_backward_traced", "mta_backward_workspace_size",
           "mta_backward_kernel_count", "mta_backward_kernel_name")


class MtaShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int),
                ("d", ctypes.c_int), ("c_q", ctypes.c_int), ("c_k", ctypes.c_int),
                ("c_h", ctypes.c_int), ("io", ctypes.c_int), ("gn_eps", ctypes.c_float)]

    def __repr__(self):
        return "MtaShape(B=%d, H=%d, T=%d, d=%d, c_q=%d, c_k=%d, c_h=%d, io=%s, gn_eps=%g)" % (
            self.B, self.H, self.T, self.d, self.c_q, self.c_k, self.c_h,
            "bf16" if self.io == MTA_BF16 else "f32", self.gn_eps)


class MtaComposition(ctypes.Structure):
    _fields_ = [("w_kq", ctypes.c_void_p), ("w_head", ctypes.c_void_p),
                ("w_kq_post", ctypes.c_void_p), ("w_head_post", ctypes.c_void_p),
                ("w_head_pre", ctypes.c_void_p), ("exact_mask", ctypes.c_int),
                ("w_kq_3d", ctypes.c_void_p)]


class MtaError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__("%s failed: %s (%d)" % (fn, STATUS.get(status, "?"), status))


_lib = None


def lib():
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libmta.so is not built (%s); run "
                               "`python -m convolved_logit_attention_b200.build`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        sp = ctypes.POINTER(MtaShape)
        vp, fp = ctypes.c_void_p, ctypes.c_void_p
        L.mta_version.argtypes, L.mta_version.restype = [], ctypes.c_int
        L.mta_status_string.argtypes, L.mta_status_string.restype = [ctypes.c_int], ctypes.c_char_p
        L.mta_forward_path.argtypes, L.mta_forward_path.restype = [sp], ctypes.c_int
        L.mta_workspace_size.argtypes, L.mta_workspace_size.restype = [sp], ctypes.c_size_t
        L.mta_unfused_workspace_size.argtypes = [sp]
        L.mta_unfused_workspace_size.restype = ctypes.c_size_t
        fwd = [sp, vp, vp, vp, fp, fp, fp, fp, ctypes.c_float, vp, vp, ctypes.c_size_t, vp]
        L.mta_forward.argtypes, L.mta_forward.restype = fwd, ctypes.c_int
        L.mta_forward_unfused.argtypes, L.mta_forward_unfused.restype = fwd, ctypes.c_int
        L.mta_debug_attention.argtypes = [sp, vp, vp, fp, fp, fp, ctypes.c_int, vp,
                                          ctypes.c_size_t, vp]
        L.mta_debug_attention.restype = ctypes.c_int
        L.mta_sync_status.argtypes, L.mta_sync_status.restype = [vp], ctypes.c_int
        L.mta_kernel_count.argtypes, L.mta_kernel_count.restype = [sp, ctypes.c_int], ctypes.c_int
        L.mta_kernel_name.argtypes = [sp, ctypes.c_int, ctypes.c_int]
        L.mta_kernel_name.restype = ctypes.c_char_p
        L.mta_forward_traced.argtypes = [ctypes.c_int] + fwd + [ctypes.POINTER(ctypes.c_void_p),
                                                               ctypes.c_int]
        L.mta_forward_traced.restype = ctypes.c_int
        L.mta_selftest_wait_timeout.argtypes = [ctypes.c_longlong, vp]
        L.mta_selftest_wait_timeout.restype = ctypes.c_int
        L.mta_forward_noalloc.argtypes = [sp, vp, vp, vp, fp, fp, fp, fp, ctypes.c_float, vp, vp]
        L.mta_forward_noalloc.restype = ctypes.c_int
        L.mta_forward_gated.argtypes = [sp, vp, vp, vp, fp, fp, fp, fp, fp, vp, vp,
                                        ctypes.c_size_t, vp]
        L.mta_forward_gated.restype = ctypes.c_int
        cp = ctypes.POINTER(MtaComposition)
        L.mta_composed_workspace_size.argtypes = [sp, cp]
        L.mta_composed_workspace_size.restype = ctypes.c_size_t
        comp = [sp, vp, vp, vp, cp, fp, fp, ctypes.c_float, fp, vp, vp, ctypes.c_size_t, vp]
        L.mta_forward_composed.argtypes, L.mta_forward_composed.restype = comp, ctypes.c_int
        L.mta_forward_composed_traced.argtypes = comp + [ctypes.POINTER(ctypes.c_void_p),
                                                         ctypes.c_int]
        L.mta_forward_composed_traced.restype = ctypes.c_int
        L.mta_composed_kernel_count.argtypes = [sp, cp]
        L.mta_composed_kernel_count.restype = ctypes.c_int
        L.mta_composed_kernel_name.argtypes = [sp, cp, ctypes.c_int]
        L.mta_composed_kernel_name.restype = ctypes.c_char_p
        bwd = [sp, vp, vp, vp, fp, fp, fp, fp, ctypes.c_float, fp, vp] + [fp] * 8 + \
            [vp, ctypes.c_size_t, vp]
        L.mta_backward.argtypes, L.mta_backward.restype = bwd, ctypes.c_int
        L.mta_backward_traced.argtypes = bwd + [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int]
        L.mta_backward_traced.restype = ctypes.c_int
        L.mta_backward_workspace_size.argtypes = [sp]
        L.mta_backward_workspace_size.restype = ctypes.c_size_t
        L.mta_backward_kernel_count.argtypes = [sp]
        L.mta_backward_kernel_count.restype = ctypes.c_int
        L.mta_backward_kernel_name.argtypes = [sp, ctypes.c_int]
        L.mta_backward_kernel_name.restype = ctypes.c_char_p
        _lib = L
    return _lib


def make_shape(B, H, T, d, c_q, c_k, c_h, io="bf16", gn_eps=1e-5) -> MtaShape:
    return MtaShape(int(B), int(H), int(T), int(d), int(c_q), int(c_k), int(c_h),
                    MTA_BF16 if io in ("bf16", torch.bfloat16) else MTA_F32, float(gn_eps))


def shape_of(q, w_kq, w_head, gn_eps=1e-5) -> MtaShape:
    B, H, T, d = q.shape
    _, c_q, c_k = w_kq.shape
    c_h = w_head.shape[-1]
    return make_shape(B, H, T, d, c_q, c_k, c_h, q.dtype, gn_eps)


def _stream_ptr(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn, status):
    if status != 0:
        raise MtaError(fn, status)


def _check_inputs(q, k, v, w_kq, w_head, gn_weight, gn_bias):
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors")
    if q.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("q, k, v must be float32 or bfloat16")
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t is None:
            continue
        if t.device != dev or t.dtype != q.dtype or t.shape != q.shape or not t.is_contiguous():
            raise ValueError("%s must be a contiguous %s tensor of shape %s on %s"
                             % (name, q.dtype, tuple(q.shape), dev))
    for name, t in (("w_kq", w_kq), ("w_head", w_head), ("gn_weight", gn_weight),
                    ("gn_bias", gn_bias)):
        if t is None:
            continue
        if t.device != dev or t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError("%s must be a contiguous float32 tensor on %s" % (name, dev))
    B, H, T, d = q.shape
    if w_kq.dim() != 3 or w_kq.shape[0] != H:
        raise ValueError("w_kq must be [H, c_q, c_k]")
    c_h = w_head.shape[-1]
    if w_head.dim() != 3 or w_head.shape[1] != c_h or c_h < 1 or H % c_h or w_head.shape[0] != H // c_h:
        raise ValueError("w_head must be [H/c_h, c_h, c_h]")
    if gn_weight is not None and (gn_weight.numel() != H * d or gn_bias.numel() != H * d):
        raise ValueError("gn_weight and gn_bias must have H*d elements")


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def mta_version() -> int:
    return lib().mta_version()


def mta_status_string(status: int) -> str:
    return lib().mta_status_string(int(status)).decode()


def mta_forward_path(shape: MtaShape) -> int:
    return lib().mta_forward_path(ctypes.byref(shape))


def mta_workspace_size(shape: MtaShape) -> int:
    return lib().mta_workspace_size(ctypes.byref(shape))


def mta_unfused_workspace_size(shape: MtaShape) -> int:
    return lib().mta_unfused_workspace_size(ctypes.byref(shape))


def _workspace(nbytes, device, workspace):
    if workspace is None:
        return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)
    if workspace.device != device or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous tensor on %s" % device)
    return workspace


def mta_kernel_count(shape: MtaShape, unfused: bool = False) -> int:
    return lib().mta_kernel_count(ctypes.byref(shape), int(bool(unfused)))


def mta_kernel_name(shape: MtaShape, index: int, unfused: bool = False) -> str:
    r = lib().mta_kernel_name(ctypes.byref(shape), int(bool(unfused)), int(index))
    return r.decode() if r is not None else None


def _after(check, stream, device):
    """With check, synchronise the call's stream and raise MtaError on a
    device-side flag (MTA_ERR_RANGE, MTA_ERR_DEVICE_TIMEOUT)."""
    if check:
        mta_sync_status(stream, device)


def _forward(fn_name, size_fn, q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale,
             out, workspace, stream, gn_eps, traced=None, check=False):
    _check_inputs(q, k, v, w_kq, w_head, gn_weight, gn_bias)
    B, H, T, d = q.shape
    if out is None:
        out = torch.empty((B, T, H * d), dtype=q.dtype, device=q.device)
    elif (out.shape != (B, T, H * d) or out.dtype != q.dtype or out.device != q.device
          or not out.is_contiguous()):
        raise ValueError("out must be a contiguous [B, T, H*d] tensor like q")
    shape = shape_of(q, w_kq, w_head, gn_eps)
    ws = _workspace(size_fn(shape), q.device, workspace)
    args = [ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(w_kq), _ptr(w_head),
            _ptr(gn_weight), _ptr(gn_bias), float(depth_scale), _ptr(out), _ptr(ws),
            ws.numel() * ws.element_size(), _stream_ptr(stream, q.device)]
    if traced is None:
        status = getattr(lib(), fn_name)(*args)
    else:
        unfused, events = traced
        handles = (ctypes.c_void_p * max(len(events), 1))(*[e.cuda_event for e in events])
        status = lib().mta_forward_traced(int(unfused), *args, handles, len(events))
    _check(fn_name, status)
    _after(check, stream, q.device)
    return out


def mta_forward(q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, out=None,
                workspace=None, stream=None, gn_eps=1e-5, check=False):
    """MTA forward on the path mta_forward_path() names; returns out [B, T, H*d].

    The call is asynchronous.  Device-side conditions (a bounded wait that
    ran out, a value outside the range of the fused path's fp16 operands)
    are only seen at a synchronisation: with check=True the call synchronises
    its stream and raises MtaError for them; otherwise call mta_sync_status()."""
    return _forward("mta_forward", mta_workspace_size, q, k, v, w_kq, w_head, gn_weight,
                    gn_bias, depth_scale, out, workspace, stream, gn_eps, check=check)


def mta_forward_gated(q, k, v, w_kq, w_head, gn_weight, gn_bias, gate, out=None,
                      workspace=None, stream=None, gn_eps=1e-5, check=False):
    """MTA forward with the sigmoid-gated output: head h of GroupNorm times
    sigmoid(gate[h]) (gate: float32 [H] on the device); returns out [B, T, H*d].
    check as for mta_forward."""
    _check_inputs(q, k, v, w_kq, w_head, gn_weight, gn_bias)
    B, H, T, d = q.shape
    if gate.dtype != torch.float32 or gate.shape != (H,) or gate.device != q.device \
            or not gate.is_contiguous():
        raise ValueError("gate must be a contiguous float32 [H] tensor on q's device")
    if out is None:
        out = torch.empty((B, T, H * d), dtype=q.dtype, device=q.device)
    elif (out.shape != (B, T, H * d) or out.dtype != q.dtype or out.device != q.device
          or not out.is_contiguous()):
        raise ValueError("out must be a contiguous [B, T, H*d] tensor like q")
    shape = shape_of(q, w_kq, w_head, gn_eps)
    ws = _workspace(mta_workspace_size(shape), q.device, workspace)
    status = lib().mta_forward_gated(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(w_kq),
                                     _ptr(w_head), _ptr(gn_weight), _ptr(gn_bias), _ptr(gate),
                                     _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                                     _stream_ptr(stream, q.device))
    _check("mta_forward_gated", status)
    _after(check, stream, q.device)
    return out


def mta_forward_unfused(q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, out=None,
                        workspace=None, stream=None, gn_eps=1e-5, check=False):
    """MTA forward with materialised fp32 T x T maps (tensor-core Q K^T and A V
    for bf16 I/O at d = 64 or 128); check as for mta_forward."""
    return _forward("mta_forward_unfused", mta_unfused_workspace_size, q, k, v, w_kq, w_head,
                    gn_weight, gn_bias, depth_scale, out, workspace, stream, gn_eps,
                    check=check)


def mta_forward_traced(unfused, events, q, k, v, w_kq, w_head, gn_weight, gn_bias,
                       depth_scale, out=None, workspace=None, stream=None, gn_eps=1e-5):
    """mta_forward (unfused=False) or mta_forward_unfused (unfused=True) that
    records the torch.cuda.Event objects in `events` around its kernel
    launches: events[2*i] before and events[2*i+1] after launch i."""
    for e in events:
        if not e.cuda_event:
            e.record()   # torch creates the underlying cudaEvent_t on first record
    size_fn = mta_unfused_workspace_size if unfused else mta_workspace_size
    return _forward("mta_forward_traced", size_fn, q, k, v, w_kq, w_head, gn_weight, gn_bias,
                    depth_scale, out, workspace, stream, gn_eps, traced=(unfused, events))


def mta_debug_attention(q, k, w_kq, w_head, stage, attn=None, workspace=None, stream=None):
    """attn [B, H, T, T] float32: pre-mix softmax (stage 0) or post-mix A_new (stage 1)."""
    _check_inputs(q, k, None, w_kq, w_head, None, None)
    B, H, T, d = q.shape
    if attn is None:
        attn = torch.empty((B, H, T, T), dtype=torch.float32, device=q.device)
    shape = shape_of(q, w_kq, w_head)
    ws = _workspace(mta_unfused_workspace_size(shape), q.device, workspace)
    status = lib().mta_debug_attention(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(w_kq),
                                       _ptr(w_head), _ptr(attn), int(stage), _ptr(ws),
                                       ws.numel() * ws.element_size(),
                                       _stream_ptr(stream, q.device))
    _check("mta_debug_attention", status)
    return attn


def mta_selftest_wait_timeout(budget_cycles=1 << 20, stream=None, device=None):
    """Enqueues the timeout-path diagnostic kernel (see include/mta.h)."""
    if device is None:
        device = torch.device("cuda", torch.cuda.current_device())
    _check("mta_selftest_wait_timeout",
           lib().mta_selftest_wait_timeout(int(budget_cycles), _stream_ptr(stream, device)))


def mta_sync_status(stream=None, device=None):
    """Synchronises the stream and raises MtaError for a device-side flag
    (MTA_ERR_DEVICE_TIMEOUT, MTA_ERR_RANGE).  The flags are one word per
    device: this reports what any work on the device raised since the last
    report."""
    if device is None:
        device = torch.device("cuda", torch.cuda.current_device())
    _check("mta_sync_status", lib().mta_sync_status(_stream_ptr(stream, device)))


def composition(w_kq=None, w_head=None, w_kq_post=None, w_head_post=None, w_head_pre=None,
                exact_mask=False, w_kq_3d=None) -> MtaComposition:
    """The C struct of a composition; the tensors must outlive its use."""
    ptrs = [t.data_ptr() if t is not None else None
            for t in (w_kq, w_head, w_kq_post, w_head_post, w_head_pre)]
    return MtaComposition(*ptrs, int(bool(exact_mask)),
                          w_kq_3d.data_ptr() if w_kq_3d is not None else None)


def composed_shape(q, w_kq=None, w_head=None, w_kq_post=None, w_head_post=None,
                   gn_eps=1e-5, w_head_pre=None, w_kq_3d=None) -> MtaShape:
    """Shape of a composition: (c_q, c_k) from the key-query kernels (equal
    when both are given), c_h from the head mixes or the 3-D kernel (1 when
    there is none)."""
    B, H, T, d = q.shape
    kq = [w for w in (w_kq, w_kq_post) if w is not None]
    hm = [w for w in (w_head_pre, w_head, w_head_post) if w is not None]
    if w_kq_3d is not None:
        if w_kq_3d.dim() != 5:
            raise ValueError("w_kq_3d must be [H/c_h, c_h, c_h, c_q, c_k]")
        c_h, c_q, c_k = tuple(w_kq_3d.shape[2:])
        if tuple(w_kq_3d.shape) != (H // c_h, c_h, c_h, c_q, c_k) or H % c_h:
            raise ValueError("w_kq_3d must be [H/c_h, c_h, c_h, c_q, c_k]")
    else:
        c_q, c_k = tuple(kq[0].shape[1:]) if kq else (1, 1)
        c_h = hm[0].shape[-1] if hm else 1
    for w in kq:
        if w.dim() != 3 or tuple(w.shape) != (H, c_q, c_k):
            raise ValueError("key-query kernels must both be [H, c_q, c_k]")
    for w in hm:
        if w.dim() != 3 or c_h < 1 or H % c_h or tuple(w.shape) != (H // c_h, c_h, c_h):
            raise ValueError("head mixes must both be [H/c_h, c_h, c_h]")
    return make_shape(B, H, T, d, c_q, c_k, c_h, q.dtype, gn_eps)


def mta_composed_kernel_names(shape: MtaShape, comp: MtaComposition):
    n = lib().mta_composed_kernel_count(ctypes.byref(shape), ctypes.byref(comp))
    return [lib().mta_composed_kernel_name(ctypes.byref(shape), ctypes.byref(comp), i).decode()
            for i in range(n)]


def mta_forward_composed(q, k, v, w_kq=None, w_head=None, w_kq_post=None, w_head_post=None,
                         gn_weight=None, gn_bias=None, depth_scale=1.0, gate=None, out=None,
                         workspace=None, stream=None, gn_eps=1e-5, events=None,
                         w_head_pre=None, exact_mask=False, w_kq_3d=None, check=False):
    """Forward of one composition of the module (see mta_composition in
    include/mta.h): weights left as None are steps left out.  gate (float32
    [H]) replaces the depth scale by sigmoid(gate[h]).  With events (a list
    of torch.cuda.Event, two per launch) the traced entry records them
    around the launches.  check as for mta_forward.  Returns out [B, T, H*d]."""
    ws_ = [w_kq, w_head, w_kq_post, w_head_post, w_head_pre, w_kq_3d]
    if q.device.type != "cuda":
        raise ValueError("inputs must be CUDA tensors")
    for name, t in (("k", k), ("v", v)):
        if t.device != q.device or t.dtype != q.dtype or t.shape != q.shape or not t.is_contiguous():
            raise ValueError("%s must be a contiguous tensor like q" % name)
    if q.dtype not in (torch.float32, torch.bfloat16) or not q.is_contiguous():
        raise ValueError("q must be a contiguous float32 or bfloat16 tensor")
    B, H, T, d = q.shape
    for t in ws_ + [gn_weight, gn_bias, gate]:
        if t is not None and (t.device != q.device or t.dtype != torch.float32
                              or not t.is_contiguous()):
            raise ValueError("weights must be contiguous float32 tensors on q's device")
    if gn_weight is None or gn_bias is None or gn_weight.numel() != H * d \
            or gn_bias.numel() != H * d:
        raise ValueError("gn_weight and gn_bias must have H*d elements")
    if gate is not None and gate.shape != (H,):
        raise ValueError("gate must be [H]")
    shape = composed_shape(q, *ws_[:4], gn_eps=gn_eps, w_head_pre=w_head_pre, w_kq_3d=w_kq_3d)
    comp = composition(*ws_[:5], exact_mask=exact_mask, w_kq_3d=w_kq_3d)
    if out is None:
        out = torch.empty((B, T, H * d), dtype=q.dtype, device=q.device)
    elif (out.shape != (B, T, H * d) or out.dtype != q.dtype or out.device != q.device
          or not out.is_contiguous()):
        raise ValueError("out must be a contiguous [B, T, H*d] tensor like q")
    need = lib().mta_composed_workspace_size(ctypes.byref(shape), ctypes.byref(comp))
    ws = _workspace(need, q.device, workspace)
    args = [ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), ctypes.byref(comp), _ptr(gn_weight),
            _ptr(gn_bias), float(depth_scale), _ptr(gate), _ptr(out), _ptr(ws),
            ws.numel() * ws.element_size(), _stream_ptr(stream, q.device)]
    if events is None:
        _check("mta_forward_composed", lib().mta_forward_composed(*args))
    else:
        for e in events:
            if not e.cuda_event:
                e.record()
        handles = (ctypes.c_void_p * max(len(events), 1))(*[e.cuda_event for e in events])
        _check("mta_forward_composed_traced",
               lib().mta_forward_composed_traced(*args, handles, len(events)))
    _after(check, stream, q.device)
    return out


GRAD_NAMES = ("q", "k", "v", "w_kq", "w_head", "gn_weight", "gn_bias")


def mta_backward_workspace_size(shape: MtaShape) -> int:
    return lib().mta_backward_workspace_size(ctypes.byref(shape))


def mta_backward_kernel_names(shape: MtaShape):
    n = lib().mta_backward_kernel_count(ctypes.byref(shape))
    return [lib().mta_backward_kernel_name(ctypes.byref(shape), i).decode() for i in range(n)]


def mta_backward(q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, dout, gate=None,
                 workspace=None, stream=None, gn_eps=1e-5, events=None, check=False):
    """Gradients of the forward (mta_forward, or mta_forward_gated with gate)
    for the upstream gradient dout [B, T, H*d] (q's dtype): a dict of float32
    tensors keyed by the input names (GRAD_NAMES, plus "gate" with a gate).
    With events (torch.cuda.Event, two per launch) the traced entry records
    them around its launches."""
    _check_inputs(q, k, v, w_kq, w_head, gn_weight, gn_bias)
    B, H, T, d = q.shape
    if (dout.shape != (B, T, H * d) or dout.dtype != q.dtype or dout.device != q.device
            or not dout.is_contiguous()):
        raise ValueError("dout must be a contiguous [B, T, H*d] tensor like q")
    if gate is not None and (gate.dtype != torch.float32 or gate.shape != (H,)
                             or gate.device != q.device or not gate.is_contiguous()):
        raise ValueError("gate must be a contiguous float32 [H] tensor on q's device")
    shape = shape_of(q, w_kq, w_head, gn_eps)
    f32 = dict(dtype=torch.float32, device=q.device)
    g = {"q": torch.empty(q.shape, **f32), "k": torch.empty(q.shape, **f32),
         "v": torch.empty(q.shape, **f32), "w_kq": torch.empty(w_kq.shape, **f32),
         "w_head": torch.empty(w_head.shape, **f32), "gn_weight": torch.empty(H * d, **f32),
         "gn_bias": torch.empty(H * d, **f32)}
    if gate is not None:
        g["gate"] = torch.empty(H, **f32)
    ws = _workspace(mta_backward_workspace_size(shape), q.device, workspace)
    args = [ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(w_kq), _ptr(w_head),
            _ptr(gn_weight), _ptr(gn_bias), float(depth_scale), _ptr(gate), _ptr(dout)]
    args += [_ptr(g[n]) for n in GRAD_NAMES] + [_ptr(g.get("gate"))]
    args += [_ptr(ws), ws.numel() * ws.element_size(), _stream_ptr(stream, q.device)]
    if events is None:
        _check("mta_backward", lib().mta_backward(*args))
    else:
        for e in events:
            if not e.cuda_event:
                e.record()
        handles = (ctypes.c_void_p * max(len(events), 1))(*[e.cuda_event for e in events])
        _check("mta_backward_traced", lib().mta_backward_traced(*args, handles, len(events)))
    _after(check, stream, q.device)
    return g
