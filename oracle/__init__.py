"""fp64 CPU oracle of the Multi-Token Attention forward pass.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke entry of the package and
the CPU-baseline leg of the benchmark are the only callers.  The CUDA library
and its Python binding never import this package.

The arithmetic lives in mta_oracle.c (plain loops in double precision, one
function per step of the pages' definition); this module only marshals numpy
arrays through ctypes.  All inputs are widened to float64 before the call.
"""
import ctypes
import os

import numpy as np

from . import build as _build


class _Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int),
                ("d", ctypes.c_int), ("c_q", ctypes.c_int), ("c_k", ctypes.c_int),
                ("c_h", ctypes.c_int), ("gn_eps", ctypes.c_double)]


class _Composition(ctypes.Structure):
    _fields_ = [("w_kq", ctypes.c_void_p), ("w_head_pre", ctypes.c_void_p),
                ("w_head", ctypes.c_void_p), ("w_kq_post", ctypes.c_void_p),
                ("w_head_post", ctypes.c_void_p), ("exact_mask", ctypes.c_int),
                ("w_kq_3d", ctypes.c_void_p)]


_lib = None


def _configure(lib):
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int)
    sp = ctypes.POINTER(_Shape)
    lib.mta_oracle_forward.argtypes = [sp, dp, dp, dp, dp, dp, dp, dp, ctypes.c_double,
                                       dp, ctypes.c_int]
    lib.mta_oracle_rows.argtypes = [sp, dp, dp, dp, dp, dp, dp, dp, ctypes.c_double,
                                    ctypes.c_int, ip, ctypes.c_int, dp, ctypes.c_int]
    lib.mta_oracle_stages.argtypes = [sp, dp, dp, dp, dp, dp, dp, dp, ctypes.c_double,
                                      ctypes.c_int, dp, dp, dp, dp, dp]
    lib.mta_oracle_forward_gated.argtypes = [sp, dp, dp, dp, dp, dp, dp, dp, dp, dp, ctypes.c_int]
    lib.mta_oracle_rows_gated.argtypes = [sp, dp, dp, dp, dp, dp, dp, dp, dp, ctypes.c_int, ip,
                                          ctypes.c_int, dp, ctypes.c_int]
    cp = ctypes.POINTER(_Composition)
    lib.mta_oracle_forward_composed.argtypes = [sp, dp, dp, dp, cp, dp, dp, ctypes.c_double, dp,
                                                dp, ctypes.c_int]
    lib.mta_oracle_rows_composed.argtypes = [sp, dp, dp, dp, cp, dp, dp, ctypes.c_double, dp,
                                             ctypes.c_int, ip, ctypes.c_int, dp, ctypes.c_int]
    lib.mta_oracle_stages_composed.argtypes = [sp, dp, dp, dp, cp, dp, dp, ctypes.c_double, dp,
                                               ctypes.c_int, dp, dp, dp, dp, dp, dp]
    lib.mta_oracle_max_threads.argtypes = []
    lib.mta_oracle_set_row_chunk.argtypes = [ctypes.c_int]
    lib.mta_oracle_set_row_chunk.restype = None
    for f in (lib.mta_oracle_forward, lib.mta_oracle_rows, lib.mta_oracle_stages,
              lib.mta_oracle_forward_gated, lib.mta_oracle_rows_gated,
              lib.mta_oracle_forward_composed, lib.mta_oracle_rows_composed,
              lib.mta_oracle_stages_composed, lib.mta_oracle_max_threads):
        f.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _configure(ctypes.CDLL(_build.build()))
    return _lib


class use_library:
    """Context manager that routes this module's calls to another build of
    the oracle source (the mutation tests use it to check that the pins
    catch planted mistakes)."""

    def __init__(self, path):
        self._new = _configure(ctypes.CDLL(path))

    def __enter__(self):
        global _lib
        self._old = _lib
        _lib = self._new
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self._old
        return False


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double)) if a is not None else None


def _shape(B, H, T, d, c_q, c_k, c_h, gn_eps):
    return _Shape(int(B), int(H), int(T), int(d), int(c_q), int(c_k), int(c_h), float(gn_eps))


def _unpack(q, w_kq, w_head):
    B, H, T, d = q.shape
    _, c_q, c_k = w_kq.shape
    c_h = w_head.shape[-1]
    return B, H, T, d, c_q, c_k, c_h


def max_threads() -> int:
    return int(_load().mta_oracle_max_threads())


def set_row_chunk(rows: int) -> None:
    """Rows per task of the full forward (0: chosen from the thread count).
    The split never changes a value; the tests use this to show it."""
    _load().mta_oracle_set_row_chunk(int(rows))


def forward(q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, gn_eps=1e-5,
            nthreads=0, gate=None):
    """out[B, T, H*d] for q, k, v [B, H, T, d], w_kq [H, c_q, c_k],
    w_head [H/c_h, c_h, c_h], gn_weight/gn_bias [H*d].  With gate [H] given,
    head h's GroupNorm output is scaled by sigmoid(gate[h]) instead of
    depth_scale (which is then ignored)."""
    q, k, v, w_kq, w_head, gw, gb = map(_f64, (q, k, v, w_kq, w_head, gn_weight, gn_bias))
    B, H, T, d, c_q, c_k, c_h = _unpack(q, w_kq, w_head)
    out = np.empty((B, T, H * d), dtype=np.float64)
    s = _shape(B, H, T, d, c_q, c_k, c_h, gn_eps)
    if gate is not None:
        g = _f64(gate)
        assert g.shape == (H,)
        rc = _load().mta_oracle_forward_gated(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v),
                                              _ptr(w_kq), _ptr(w_head), _ptr(gw), _ptr(gb),
                                              _ptr(g), _ptr(out), int(nthreads))
    else:
        rc = _load().mta_oracle_forward(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(w_kq),
                                        _ptr(w_head), _ptr(gw), _ptr(gb), float(depth_scale),
                                        _ptr(out), int(nthreads))
    if rc != 0:
        raise RuntimeError("mta_oracle_forward failed (%d)" % rc)
    return out


def rows(q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, b, row_idx,
         gn_eps=1e-5, nthreads=0, gate=None):
    """out[b, row_idx, :] computed one row at a time: [len(row_idx), H*d]
    (gate as in forward)."""
    q, k, v, w_kq, w_head, gw, gb = map(_f64, (q, k, v, w_kq, w_head, gn_weight, gn_bias))
    B, H, T, d, c_q, c_k, c_h = _unpack(q, w_kq, w_head)
    idx = np.ascontiguousarray(np.asarray(row_idx, dtype=np.int32))
    out = np.empty((idx.size, H * d), dtype=np.float64)
    s = _shape(B, H, T, d, c_q, c_k, c_h, gn_eps)
    ip = idx.ctypes.data_as(ctypes.POINTER(ctypes.c_int))
    if gate is not None:
        g = _f64(gate)
        assert g.shape == (H,)
        rc = _load().mta_oracle_rows_gated(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(w_kq),
                                           _ptr(w_head), _ptr(gw), _ptr(gb), _ptr(g), int(b), ip,
                                           int(idx.size), _ptr(out), int(nthreads))
    else:
        rc = _load().mta_oracle_rows(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(w_kq),
                                     _ptr(w_head), _ptr(gw), _ptr(gb), float(depth_scale), int(b),
                                     ip, int(idx.size), _ptr(out), int(nthreads))
    if rc != 0:
        raise RuntimeError("mta_oracle_rows failed (%d)" % rc)
    return out


def stages(q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, b=0, gn_eps=1e-5):
    """Intermediates of batch entry b (small T only), as a dict:
    C [H,T,T] conv logits after both masks (-inf above the diagonal),
    P [H,T,T] pre-mix softmax, A [H,T,T] post-mix attention,
    O [H,T,d] pre-normalisation head outputs, out [T, H*d]."""
    q, k, v, w_kq, w_head, gw, gb = map(_f64, (q, k, v, w_kq, w_head, gn_weight, gn_bias))
    B, H, T, d, c_q, c_k, c_h = _unpack(q, w_kq, w_head)
    C = np.empty((H, T, T)); P = np.empty((H, T, T)); A = np.empty((H, T, T))
    O = np.empty((H, T, d)); out = np.empty((T, H * d))
    s = _shape(B, H, T, d, c_q, c_k, c_h, gn_eps)
    rc = _load().mta_oracle_stages(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v), _ptr(w_kq),
                                   _ptr(w_head), _ptr(gw), _ptr(gb), float(depth_scale), int(b),
                                   _ptr(C), _ptr(P), _ptr(A), _ptr(O), _ptr(out))
    if rc != 0:
        raise RuntimeError("mta_oracle_stages failed (%d)" % rc)
    return {"C": C, "P": P, "A": A, "O": O, "out": out}


def _composed(q, ws, exact_mask, gn_eps, w3=None):
    """Shape and C struct of a composition.  ws = (w_kq, w_head_pre, w_head,
    w_kq_post, w_head_post), float64 arrays or None, and w3 the 3-D kernel
    [H/c_h, c_h, c_h, c_q, c_k] or None: (c_q, c_k) from the key-query
    kernels (all alike), c_h from the head mixes or the 3-D kernel (1 when
    there is none)."""
    B, H, T, d = q.shape
    kq = [w for w in (ws[0], ws[3]) if w is not None]
    hm = [w for w in (ws[1], ws[2], ws[4]) if w is not None]
    if w3 is not None:
        c_h, c_q, c_k = w3.shape[2:]
    else:
        c_q, c_k = kq[0].shape[1:] if kq else (1, 1)
        c_h = hm[0].shape[-1] if hm else 1
    for w in kq:
        assert w.shape == (H, c_q, c_k), w.shape
    for w in hm:
        assert w.shape == (H // c_h, c_h, c_h), w.shape
    if w3 is not None:
        assert w3.shape == (H // c_h, c_h, c_h, c_q, c_k), w3.shape
    comp = _Composition(*[None if w is None else w.ctypes.data for w in ws],
                        int(bool(exact_mask)), None if w3 is None else w3.ctypes.data)
    return _shape(B, H, T, d, c_q, c_k, c_h, gn_eps), comp


def _weights(w_kq, w_head_pre, w_head, w_kq_post, w_head_post):
    return [None if w is None else _f64(w)
            for w in (w_kq, w_head_pre, w_head, w_kq_post, w_head_post)]


def forward_composed(q, k, v, w_kq, w_head, w_kq_post, w_head_post, gn_weight, gn_bias,
                     depth_scale, gn_eps=1e-5, nthreads=0, gate=None, w_head_pre=None,
                     exact_mask=False, w_kq_3d=None):
    """out[B, T, H*d] of a composition of "Putting Everything Together": the
    steps Mask_0, [key-query conv w_kq], [head mix of the logits
    w_head_pre], Mask_-inf, softmax, [head mix w_head], [key-query conv
    w_kq_post on the probabilities, Mask_0], [head mix w_head_post], A V,
    GroupNorm, scale; a bracketed step whose weights are None is left out.
    exact_mask: the w_kq conv uses Eq. (4)'s indicator instead of Mask_0.
    w_kq_3d [H/c_h, c_h, c_h, c_q, c_k]: the 3-D conv over (query, key,
    head) in place of w_kq.  gate as in forward."""
    q, k, v, gw, gb = map(_f64, (q, k, v, gn_weight, gn_bias))
    ws = _weights(w_kq, w_head_pre, w_head, w_kq_post, w_head_post)
    w3 = None if w_kq_3d is None else _f64(w_kq_3d)
    s, comp = _composed(q, ws, exact_mask, gn_eps, w3)
    g = None if gate is None else _f64(gate)
    out = np.empty((s.B, s.T, s.H * s.d), dtype=np.float64)
    rc = _load().mta_oracle_forward_composed(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v),
                                             ctypes.byref(comp), _ptr(gw), _ptr(gb),
                                             float(depth_scale), _ptr(g), _ptr(out),
                                             int(nthreads))
    if rc != 0:
        raise RuntimeError("mta_oracle_forward_composed failed (%d)" % rc)
    return out


def rows_composed(q, k, v, w_kq, w_head, w_kq_post, w_head_post, gn_weight, gn_bias,
                  depth_scale, b, row_idx, gn_eps=1e-5, nthreads=0, gate=None,
                  w_head_pre=None, exact_mask=False, w_kq_3d=None):
    """out[b, row_idx, :] of forward_composed, one row at a time."""
    q, k, v, gw, gb = map(_f64, (q, k, v, gn_weight, gn_bias))
    ws = _weights(w_kq, w_head_pre, w_head, w_kq_post, w_head_post)
    w3 = None if w_kq_3d is None else _f64(w_kq_3d)
    s, comp = _composed(q, ws, exact_mask, gn_eps, w3)
    g = None if gate is None else _f64(gate)
    idx = np.ascontiguousarray(np.asarray(row_idx, dtype=np.int32))
    out = np.empty((idx.size, s.H * s.d), dtype=np.float64)
    rc = _load().mta_oracle_rows_composed(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v),
                                          ctypes.byref(comp), _ptr(gw), _ptr(gb),
                                          float(depth_scale), _ptr(g), int(b),
                                          idx.ctypes.data_as(ctypes.POINTER(ctypes.c_int)),
                                          int(idx.size), _ptr(out), int(nthreads))
    if rc != 0:
        raise RuntimeError("mta_oracle_rows_composed failed (%d)" % rc)
    return out


def stages_composed(q, k, v, w_kq, w_head, w_kq_post, w_head_post, gn_weight, gn_bias,
                    depth_scale, b=0, gn_eps=1e-5, gate=None, w_head_pre=None,
                    exact_mask=False, w_kq_3d=None):
    """Intermediates of forward_composed for batch entry b (small T only):
    C [H,T,T] softmax input (after both masks and the logit mix), P [H,T,T]
    softmax, A1 [H,T,T] after the first head mix, A [H,T,T] the attention
    that meets V, O [H,T,d] pre-normalisation head outputs, out [T, H*d]."""
    q, k, v, gw, gb = map(_f64, (q, k, v, gn_weight, gn_bias))
    ws = _weights(w_kq, w_head_pre, w_head, w_kq_post, w_head_post)
    w3 = None if w_kq_3d is None else _f64(w_kq_3d)
    s, comp = _composed(q, ws, exact_mask, gn_eps, w3)
    g = None if gate is None else _f64(gate)
    H, T, d = s.H, s.T, s.d
    C, P, A1, A = (np.empty((H, T, T)) for _ in range(4))
    O = np.empty((H, T, d)); out = np.empty((T, H * d))
    rc = _load().mta_oracle_stages_composed(ctypes.byref(s), _ptr(q), _ptr(k), _ptr(v),
                                            ctypes.byref(comp), _ptr(gw), _ptr(gb),
                                            float(depth_scale), _ptr(g), int(b), _ptr(C),
                                            _ptr(P), _ptr(A1), _ptr(A), _ptr(O), _ptr(out))
    if rc != 0:
        raise RuntimeError("mta_oracle_stages_composed failed (%d)" % rc)
    return {"C": C, "P": P, "A1": A1, "A": A, "O": O, "out": out}
