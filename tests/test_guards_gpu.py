"""Out-of-bounds stores: canary bytes around every buffer a call writes.

compute-sanitizer is not available on the machines these tests run on, so
this is the check that the kernels' stores stay inside their buffers: the
output tensor sits between two guard regions filled with a known byte
pattern, the workspace is followed by a guard region, and after the call
every guard byte must be unchanged.  The shapes are the ragged ones where an
indexing slip would land outside: T not a multiple of the 128-row tile,
T = 1, odd numbers of query blocks (whose pair partner is padding), head
groups split over two work items, and the materialised chain.
"""
import ctypes

import numpy as np
import pytest
import torch

import convolved_logit_attention_b200 as mta
from convolved_logit_attention_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu

GUARD = 1 << 16      # bytes before and after each guarded buffer (keeps 256-B alignment)
PATTERN = 0xA5

SHAPES = [
    # B, H, T, d, c_q, c_k, c_h
    (1, 2, 1, 128, 6, 11, 2),       # a single token: one block, its partner is padding
    (1, 2, 1, 64, 6, 11, 2),
    (2, 2, 129, 128, 6, 11, 2),     # one row past a tile
    (1, 4, 200, 64, 4, 15, 2),
    (1, 2, 383, 128, 8, 15, 2),     # three blocks: an odd count, the last pair half padding
    (2, 4, 130, 128, 6, 11, 4),     # head group split over two work items
    (1, 8, 255, 64, 3, 5, 8),
    (1, 2, 513, 128, 2, 3, 1),
]
# fp32 I/O: the fused CUDA-core kernel (path 2) and, past c_h * d = 256, the chain
SHAPES_F32 = [
    (1, 4, 128, 32, 6, 11, 2),
    (2, 2, 77, 64, 4, 15, 2),
    (1, 2, 1, 128, 8, 15, 2),
]


@pytest.fixture(scope="module", autouse=True)
def _built():
    from convolved_logit_attention_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _inputs(shape, seed, io="bf16"):
    B, H, T, d, c_q, c_k, c_h = shape
    x = make_inputs(Workload("guards", B, H, T, d, c_q, c_k, c_h, io, seed=seed))
    dev = torch.device("cuda", 0)
    dt = torch.bfloat16 if io == "bf16" else torch.float32
    t = {n: torch.from_numpy(x[n]).to(dev).to(dt) for n in ("q", "k", "v")}
    for n in ("w_kq", "w_head", "gn_weight", "gn_bias"):
        t[n] = torch.from_numpy(x[n]).to(dev)
    return x, t


def _guarded(nbytes):
    """A byte buffer [guard | body | guard] filled with the pattern; returns
    (buffer, body view)."""
    buf = torch.full((GUARD + nbytes + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
    return buf, buf[GUARD:GUARD + nbytes]


def _guards_intact(buf, nbytes):
    head = buf[:GUARD]
    tail = buf[GUARD + nbytes:]
    return bool((head == PATTERN).all()) and bool((tail == PATTERN).all())


@pytest.mark.parametrize("unfused", [0, 1], ids=["fused", "materialised"])
@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_stores_stay_inside_out_and_workspace(shape, unfused):
    B, H, T, d, c_q, c_k, c_h = shape
    x, t = _inputs(shape, seed=sum(shape))
    mshape = mta.make_shape(B, H, T, d, c_q, c_k, c_h, "bf16", x["gn_eps"])
    if not unfused:
        assert mta.mta_forward_path(mshape) == mta.MTA_PATH_FUSED_TC
    need = (mta.mta_unfused_workspace_size(mshape) if unfused
            else mta.mta_workspace_size(mshape))
    out_bytes = B * T * H * d * 2
    out_buf, out_body = _guarded(out_bytes)
    ws_buf, ws_body = _guarded(need)
    L = mta.lib()
    p = lambda a: ctypes.c_void_p(a.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    fn = L.mta_forward_unfused if unfused else L.mta_forward
    rc = fn(ctypes.byref(mshape), p(t["q"]), p(t["k"]), p(t["v"]), p(t["w_kq"]), p(t["w_head"]),
            p(t["gn_weight"]), p(t["gn_bias"]), ctypes.c_float(x["depth_scale"]), p(out_body),
            p(ws_body), ctypes.c_size_t(need), stream)
    assert rc == 0
    mta.mta_sync_status()
    assert _guards_intact(out_buf, out_bytes), "a store landed outside out"
    assert _guards_intact(ws_buf, need), "a store landed outside the workspace"
    # the output itself was written everywhere (no pattern bytes left as bf16
    # 0xA5A5 = -2.87e-16 would be an implausible exact value) and is finite
    out = out_body.view(torch.bfloat16).float()
    assert torch.isfinite(out).all()
    assert not bool((out_body.view(torch.int16) == np.int16(-23131)).any())


@pytest.mark.parametrize("shape", SHAPES_F32, ids=[str(s) for s in SHAPES_F32])
def test_fp32_fused_stores_stay_inside_out(shape):
    B, H, T, d, c_q, c_k, c_h = shape
    x, t = _inputs(shape, seed=sum(shape) + 1, io="f32")
    mshape = mta.make_shape(B, H, T, d, c_q, c_k, c_h, "f32", x["gn_eps"])
    assert mta.mta_forward_path(mshape) == mta.MTA_PATH_FUSED_F32
    assert mta.mta_workspace_size(mshape) == 0
    out_bytes = B * T * H * d * 4
    out_buf, out_body = _guarded(out_bytes)
    L = mta.lib()
    p = lambda a: ctypes.c_void_p(a.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = L.mta_forward(ctypes.byref(mshape), p(t["q"]), p(t["k"]), p(t["v"]), p(t["w_kq"]),
                       p(t["w_head"]), p(t["gn_weight"]), p(t["gn_bias"]),
                       ctypes.c_float(x["depth_scale"]), p(out_body), None, ctypes.c_size_t(0),
                       stream)
    assert rc == 0
    mta.mta_sync_status()
    assert _guards_intact(out_buf, out_bytes), "a store landed outside out"
    assert torch.isfinite(out_body.view(torch.float32)).all()


# The backward pass: every gradient buffer and the workspace between guard
# regions, at ragged T, both I/O types and d = 64 / 128 (the tensor-core
# products) as well as d = 32 (the CUDA-core ones).
BWD_SHAPES = [
    # B, H, T, d, c_q, c_k, c_h, io
    (1, 2, 1, 128, 6, 11, 2, "bf16"),
    (1, 2, 129, 128, 6, 11, 2, "bf16"),
    (2, 4, 200, 64, 4, 15, 2, "f32"),
    (1, 4, 130, 128, 8, 15, 4, "bf16"),
    (1, 2, 65, 32, 3, 4, 2, "bf16"),
]


@pytest.mark.parametrize("shape", BWD_SHAPES, ids=[str(s) for s in BWD_SHAPES])
def test_backward_stores_stay_inside_gradients_and_workspace(shape):
    B, H, T, d, c_q, c_k, c_h, io = shape
    x, t = _inputs(shape[:7], seed=sum(shape[:7]) + 2, io=io)
    dt = torch.bfloat16 if io == "bf16" else torch.float32
    dout = torch.randn(B, T, H * d, device="cuda").to(dt)
    mshape = mta.make_shape(B, H, T, d, c_q, c_k, c_h, io, x["gn_eps"])
    sizes = {"q": B * H * T * d, "k": B * H * T * d, "v": B * H * T * d, "w_kq": H * c_q * c_k,
             "w_head": (H // c_h) * c_h * c_h, "gn_weight": H * d, "gn_bias": H * d}
    bufs = {n: _guarded(4 * m) for n, m in sizes.items()}
    need = mta.mta_backward_workspace_size(mshape)
    ws_buf, ws_body = _guarded(need)
    L = mta.lib()
    p = lambda a: ctypes.c_void_p(a.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = L.mta_backward(ctypes.byref(mshape), p(t["q"]), p(t["k"]), p(t["v"]), p(t["w_kq"]),
                        p(t["w_head"]), p(t["gn_weight"]), p(t["gn_bias"]),
                        ctypes.c_float(x["depth_scale"]), None, p(dout),
                        *[p(bufs[n][1]) for n in mta.GRAD_NAMES], None, p(ws_body),
                        ctypes.c_size_t(need), stream)
    assert rc == 0
    mta.mta_sync_status()
    for n, (buf, body) in bufs.items():
        assert _guards_intact(buf, 4 * sizes[n]), "a store landed outside d" + n
        assert torch.isfinite(body.view(torch.float32)).all(), "d" + n + " not finite"
    assert _guards_intact(ws_buf, need), "a store landed outside the workspace"
