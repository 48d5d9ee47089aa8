"""Parity of the CUDA backward pass (mta_backward, through the C ABI) with the
fp64 gradient oracle (oracle/backward.py), element by element.

The backward computes every step in fp32 on the materialised chain, from the
same rounded inputs and upstream gradient the oracle widens to fp64.  Its
error is fp32 rounding accumulated over sums of up to T * c_q * c_k terms,
relative to the size of the gradient, so each gradient is held to
    max-abs <= 2e-4 * S   and   rel-L2 <= 1e-4,
about two orders of magnitude above what fp32 summation of these lengths
gives on random data, and far below what a wrong index, sign or mask would
leave (those move whole rows or taps by O(1) relative error).  S is the
gradient's own largest |entry|, but at least 1% of the largest entry of any
gradient of the case: a gradient whose exact value cancels to almost zero
(dw_head at T = 1 is exactly 0, because GroupNorm's backward projects dO off
V) keeps the fp32 rounding of the terms that cancel, whose size is that of
the case's other gradients.  Such a gradient is held to the max-abs bound.
"""
import zlib

import numpy as np
import pytest
import torch

import convolved_logit_attention_b200 as mta
from convolved_logit_attention_b200.workloads import WORKLOADS, Workload, make_inputs
from oracle import backward as oracle_bwd

pytestmark = pytest.mark.gpu

TOL_REL_MAX = 2e-4
TOL_REL_L2 = 1e-4
GATE = np.array([-2.0, -0.5, 0.25, 1.5, 3.0, -1.0, 0.0, 0.75] * 4, dtype=np.float32)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from convolved_logit_attention_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _round_io(a, io):
    """The values the device sees: bf16 I/O rounds to bf16 (ties to even)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).float().numpy() if io == "bf16" else t.numpy()


def _device(x, io, dout, gate=None):
    dt = torch.bfloat16 if io == "bf16" else torch.float32
    dev = torch.device("cuda", 0)
    d = {n: torch.from_numpy(np.ascontiguousarray(x[n])).to(dev).to(dt) for n in ("q", "k", "v")}
    for n in ("w_kq", "w_head", "gn_weight", "gn_bias"):
        d[n] = torch.from_numpy(np.ascontiguousarray(x[n])).to(dev)
    d["dout"] = torch.from_numpy(np.ascontiguousarray(dout, dtype=np.float32)).to(dev).to(dt)
    d["gate"] = None if gate is None else torch.from_numpy(gate).to(dev)
    return d


def _gpu_grads(d, x):
    g = mta.mta_backward(d["q"], d["k"], d["v"], d["w_kq"], d["w_head"], d["gn_weight"],
                         d["gn_bias"], x["depth_scale"], d["dout"], gate=d["gate"],
                         gn_eps=x["gn_eps"], check=True)
    return {n: t.cpu().numpy().astype(np.float64) for n, t in g.items()}


FLOOR = 1e-2      # of the case's largest gradient entry (see the module docstring)


def assert_grads_close(got, ref, what):
    assert set(got) == set(ref), (sorted(got), sorted(ref))
    case_max = max(float(np.abs(r).max()) for r in ref.values())
    for n in ref:
        a, r = got[n], ref[n]
        assert a.shape == r.shape, (what, n, a.shape, r.shape)
        assert np.isfinite(a).all(), "%s d%s: non-finite" % (what, n)
        own = float(np.abs(r).max())
        scale = max(own, FLOOR * case_max)
        err = np.abs(a - r)
        rel_max = float(err.max()) / scale
        idx = np.unravel_index(int(err.argmax()), err.shape)
        assert rel_max <= TOL_REL_MAX, \
            "%s d%s: max-abs/S %.3g (worst at %s; max|ref| %.3g, S %.3g)" % (
                what, n, rel_max, idx, own, scale)
        if own >= FLOOR * case_max:
            rel_l2 = float(np.linalg.norm(a - r) / np.linalg.norm(r))
            assert rel_l2 <= TOL_REL_L2, "%s d%s: rel-L2 %.3g" % (what, n, rel_l2)


def _case(w, seed_dout, gate=None, x=None):
    x = make_inputs(w) if x is None else x
    rng = np.random.default_rng(seed_dout)
    dout = _round_io(rng.standard_normal((w.B, w.T, w.H * w.d)), w.io)
    d = _device(x, w.io, dout, gate)
    got = _gpu_grads(d, x)
    ref = oracle_bwd.gradients(x, dout, x["depth_scale"], gn_eps=x["gn_eps"], gate=gate)
    return got, ref


@pytest.mark.parametrize("gated", [False, True], ids=["depth", "gate"])
@pytest.mark.parametrize("name", ["tiny_f32", "toy_letters"])
def test_small_workloads_every_gradient(name, gated):
    w = WORKLOADS[name]
    gate = GATE[:w.H].copy() if gated else None
    got, ref = _case(w, 101, gate)
    assert_grads_close(got, ref, name + (" gated" if gated else ""))


RAGGED = [
    # B, H, T, d, c_q, c_k, c_h, io
    (1, 2, 1, 32, 6, 11, 2, "bf16"),        # a single token
    (2, 4, 65, 32, 3, 4, 4, "bf16"),        # even c_k, ragged T
    (1, 4, 200, 64, 6, 11, 2, "f32"),
    (1, 2, 257, 128, 2, 3, 1, "bf16"),
    (1, 8, 130, 16, 1, 1, 8, "f32"),        # 1 x 1 kernel, c_h = 8
    (1, 4, 129, 128, 8, 15, 4, "bf16"),
]


@pytest.mark.parametrize("shape", RAGGED, ids=[str(s) for s in RAGGED])
def test_ragged_shapes_every_gradient(shape):
    B, H, T, d, c_q, c_k, c_h, io = shape
    w = Workload("bwd_ragged", B, H, T, d, c_q, c_k, c_h, io,
                 seed=zlib.crc32(repr(shape).encode()) % 1000)
    got, ref = _case(w, 102)
    assert_grads_close(got, ref, str(shape))


def test_strong_kernels_and_gate():
    # kernels far from the identity: every tap and both mixing weights matter
    w = Workload("bwd_strong", 2, 4, 160, 64, 6, 11, 2, "bf16", seed=17)
    x = make_inputs(w)
    rng = np.random.default_rng(18)
    x["w_kq"] = (0.4 * rng.standard_normal(x["w_kq"].shape)).astype(np.float32)
    x["w_head"] = rng.standard_normal(x["w_head"].shape).astype(np.float32)
    got, ref = _case(w, 103, GATE[:w.H].copy(), x=x)
    assert_grads_close(got, ref, "strong gated")


def test_repeated_calls_give_identical_bits():
    w = WORKLOADS["toy_letters"]
    x = make_inputs(w)
    dout = _round_io(np.random.default_rng(104).standard_normal((w.B, w.T, w.H * w.d)), w.io)
    d = _device(x, w.io, dout)
    a = _gpu_grads(d, x)
    b = _gpu_grads(d, x)
    for n in a:
        assert np.array_equal(a[n], b[n]), n


def test_full_size_gradient_of_selected_rows():
    """The T = 4096 workload (three 2.1 GB maps in the workspace) with an
    upstream gradient that is zero except on a few rows, including both ends
    and tile edges: every element of every gradient against the oracle's
    gradient through those rows (oracle.backward.gradients_rows)."""
    w = WORKLOADS["longctx_4k"]
    x = make_inputs(w)
    rows = [0, 1, 127, 128, 2049, 4095]
    rng = np.random.default_rng(105)
    dout = np.zeros((w.B, w.T, w.H * w.d), dtype=np.float32)
    dout[:, rows] = _round_io(rng.standard_normal((w.B, len(rows), w.H * w.d)), w.io)
    d = _device(x, w.io, dout)
    got = _gpu_grads(d, x)
    del d
    torch.cuda.empty_cache()
    ref = oracle_bwd.gradients_rows(x, rows, dout[:, rows], x["depth_scale"], gn_eps=x["gn_eps"])
    assert_grads_close(got, ref, "longctx_4k rows %s" % rows)


def test_rejects_gate_without_dgate_and_bad_alignment():
    import ctypes
    w = Workload("bwd_args", 1, 2, 64, 32, 6, 11, 2, "bf16", seed=1)
    x = make_inputs(w)
    d = _device(x, w.io, np.zeros((1, 64, 64), dtype=np.float32), GATE[:2].copy())
    shape = mta.shape_of(d["q"], d["w_kq"], d["w_head"])
    L = mta.lib()
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    g = torch.zeros(1 << 20, dtype=torch.float32, device="cuda")
    ws = torch.empty(mta.mta_backward_workspace_size(shape), dtype=torch.uint8, device="cuda")
    base = [ctypes.byref(shape)] + [p(d[n]) for n in ("q", "k", "v", "w_kq", "w_head",
                                                       "gn_weight", "gn_bias")]
    grads = [p(g)] * 7
    # a gate but no dgate
    assert L.mta_backward(*base, ctypes.c_float(0.8), p(d["gate"]), p(d["dout"]), *grads, None,
                          p(ws), ctypes.c_size_t(ws.numel()), None) == -1
    # a misaligned gradient pointer
    bad = ctypes.c_void_p(g.data_ptr() + 4)
    assert L.mta_backward(*base, ctypes.c_float(0.8), None, p(d["dout"]), bad, *grads[1:],
                          None, p(ws), ctypes.c_size_t(ws.numel()), None) == -3
    # workspace too small
    assert L.mta_backward(*base, ctypes.c_float(0.8), None, p(d["dout"]), *grads, None, p(ws),
                          ctypes.c_size_t(ws.numel() - 256), None) == -4
