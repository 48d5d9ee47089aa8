"""Parity of the compositions of "Putting Everything Together: The Full MTA
Module" (with the post-softmax variant of "Key-Query Convolution", the
pre-softmax head mix of "Head Mixing Convolution" and the exact indicator of
Eq. (4)) on the GPU,
called through mta_forward_composed, against the fp64 oracle's composed
forward on the same inputs.

Tolerances as for the default forward: fp32 I/O max-abs <= 1e-4; bf16 I/O
max-abs <= 2e-2 and relative L2 <= 5e-3, on `out`.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
import convolved_logit_attention_b200 as mta
from convolved_logit_attention_b200.workloads import (COMPOSITIONS, WORKLOADS, Workload,
                                                      composed_inputs)
from tests.test_parity_gpu import assert_close
from tests.test_parity_full_gpu import assert_every_element

pytestmark = pytest.mark.gpu

WEIGHTS = ("w_kq", "w_head", "w_kq_post", "w_head_post")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from convolved_logit_attention_b200 import build
    build.build()
    assert torch.cuda.is_available()


def to_device(x, io):
    dt = torch.bfloat16 if io == "bf16" else torch.float32
    dev = torch.device("cuda", 0)
    d = {n: torch.from_numpy(np.ascontiguousarray(x[n])).to(dev).to(dt) for n in ("q", "k", "v")}
    for n in WEIGHTS + ("w_head_pre", "w_kq_3d", "gn_weight", "gn_bias"):
        d[n] = None if x[n] is None else torch.from_numpy(np.ascontiguousarray(x[n])).to(dev)
    return d


def run(d, x, gate=None, events=None):
    out = mta.mta_forward_composed(d["q"], d["k"], d["v"], *(d[n] for n in WEIGHTS),
                                   gn_weight=d["gn_weight"], gn_bias=d["gn_bias"],
                                   depth_scale=x["depth_scale"], gate=gate,
                                   gn_eps=x["gn_eps"], events=events, w_head_pre=d["w_head_pre"],
                                   exact_mask=x["exact_mask"], w_kq_3d=d["w_kq_3d"])
    mta.mta_sync_status()
    return out.float().cpu().numpy().astype(np.float64)


def oracle_full(x, gate=None):
    return oracle.forward_composed(x["q"], x["k"], x["v"], *(x[n] for n in WEIGHTS),
                                   x["gn_weight"], x["gn_bias"], x["depth_scale"],
                                   gn_eps=x["gn_eps"], gate=gate, w_head_pre=x["w_head_pre"],
                                   exact_mask=x["exact_mask"], w_kq_3d=x["w_kq_3d"])


@pytest.mark.parametrize("comp", sorted(COMPOSITIONS))
@pytest.mark.parametrize("name", ["tiny_f32", "toy_letters"])
def test_compositions_elementwise(name, comp):
    w = WORKLOADS[name]
    x = composed_inputs(w, comp)
    got = run(to_device(x, w.io), x)
    assert_close(got, oracle_full(x), w.io, "%s/%s" % (name, comp))


RAGGED = [
    # B, H, T, d, c_q, c_k, c_h, io
    (1, 2, 1, 32, 6, 11, 2, "bf16"),        # a single token
    (1, 2, 7, 64, 6, 11, 2, "f32"),         # T shorter than the kernel
    (2, 4, 65, 32, 3, 4, 4, "bf16"),        # even c_k, ragged T
    (1, 2, 257, 128, 8, 15, 2, "f32"),      # the largest kernel, ragged tiles
    (1, 8, 130, 16, 1, 1, 8, "bf16"),       # 1 x 1 kernels, c_h = 8
    (1, 16, 96, 32, 2, 3, 16, "f32"),       # c_h = 16
    (1, 2, 141, 24, 5, 9, 2, "f32"),        # d = 24: a ragged contraction chunk
    (1, 2, 77, 8, 3, 5, 1, "bf16"),         # the smallest d
]


@pytest.mark.parametrize("comp", ["repeat", "post_kq", "both_post", "exact_both_pre",
                                  "exact_repeat", "conv3d_exact_mix"])
@pytest.mark.parametrize("shape", RAGGED, ids=[str(s) for s in RAGGED])
def test_ragged_shapes_elementwise(shape, comp):
    B, H, T, d, c_q, c_k, c_h, io = shape
    w = Workload("ragged", B, H, T, d, c_q, c_k, c_h, io,
                 seed=zlib.crc32(repr(shape).encode()) % 1000)
    x = composed_inputs(w, comp)
    got = run(to_device(x, io), x)
    assert_close(got, oracle_full(x), io, "%s/%s" % (shape, comp))


def test_strong_post_kernels_and_gate():
    """Post-softmax kernels far from the identity, and the sigmoid gate."""
    w = Workload("strong", 2, 4, 160, 64, 6, 11, 2, "bf16", seed=31)
    x = composed_inputs(w, "repeat")
    rng = np.random.default_rng(32)
    x["w_kq_post"] = (0.4 * rng.standard_normal(x["w_kq_post"].shape)).astype(np.float32)
    x["w_head_post"] = rng.standard_normal(x["w_head_post"].shape).astype(np.float32)
    d = to_device(x, w.io)
    assert_close(run(d, x), oracle_full(x), w.io, "strong")
    gate = np.array([-2.0, -0.5, 0.75, 3.0], dtype=np.float32)
    got = run(d, x, gate=torch.from_numpy(gate).cuda())
    assert_close(got, oracle_full(x, gate=gate), w.io, "strong gated")


@pytest.mark.parametrize("comp", ["exact_both_pre", "exact_repeat"])
def test_strong_kernels_exact_mask_and_logit_mix(comp):
    """Kernels far from the identity in fp32, where the exact indicator of
    Eq. (4) and the logit mix move the output far beyond the tolerance: the
    GPU must match the oracle with them, and the oracle without the exact
    mask must be far off (so that the test tells the two maskings apart)."""
    w = Workload("strong_exact", 2, 4, 160, 64, 6, 11, 2, "f32", seed=33)
    x = composed_inputs(w, comp)
    rng = np.random.default_rng(34)
    x["w_kq"] = (0.4 * rng.standard_normal(x["w_kq"].shape)).astype(np.float32)
    if x["w_head_pre"] is not None:
        x["w_head_pre"] = rng.standard_normal(x["w_head_pre"].shape).astype(np.float32)
    got = run(to_device(x, w.io), x)
    ref = oracle_full(x)
    assert_close(got, ref, w.io, "strong " + comp)
    two_pass = oracle_full(dict(x, exact_mask=False))
    assert np.abs(two_pass - ref).max() > 100 * 1e-4


def test_strong_conv3d_kernel():
    """A 3-D kernel far from the identity, cross-head taps included, in
    fp32 with the exact mask and without."""
    w = Workload("strong_3d", 2, 4, 150, 32, 4, 7, 2, "f32", seed=35)
    rng = np.random.default_rng(36)
    for comp in ("conv3d", "conv3d_exact_mix"):
        x = composed_inputs(w, comp)
        x["w_kq_3d"] = (0.4 * rng.standard_normal(x["w_kq_3d"].shape)).astype(np.float32)
        assert_close(run(to_device(x, w.io), x), oracle_full(x), w.io, "strong " + comp)


def test_default_composition_is_mta_forward():
    """The default composition takes mta_forward's own path: same bits."""
    w = WORKLOADS["toy_letters"]
    x = composed_inputs(w, "default")
    d = to_device(x, w.io)
    got = run(d, x)
    ref = mta.mta_forward(d["q"], d["k"], d["v"], d["w_kq"], d["w_head"], d["gn_weight"],
                          d["gn_bias"], x["depth_scale"], gn_eps=x["gn_eps"])
    mta.mta_sync_status()
    assert np.array_equal(got, ref.float().cpu().numpy().astype(np.float64))


def test_traced_launches_follow_the_chain():
    w = WORKLOADS["tiny_f32"]
    x = composed_inputs(w, "repeat")
    d = to_device(x, w.io)
    shape = mta.composed_shape(d["q"], *(d[n] for n in WEIGHTS))
    names = mta.mta_composed_kernel_names(shape, mta.composition(*(d[n] for n in WEIGHTS)))
    assert names == ["k_logits", "k_conv", "k_softmax_mix", "k_conv", "k_head_mix",
                     "k_pv_groupnorm"]
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * len(names))]
    got = run(d, x, events=ev)
    torch.cuda.synchronize()
    times = [ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(len(names))]
    assert all(t > 0 for t in times)
    assert_close(got, oracle_full(x), w.io, "traced")


@pytest.mark.parametrize("comp", ["exact", "repeat", "both_post", "exact_both_pre", "conv3d"])
def test_full_size_every_element(comp):
    """The T = 4096 workload (two [B,H,T,T] fp32 maps, 4.3 GB), every element
    against the oracle's full forward of the same composition."""
    w = WORKLOADS["longctx_4k"]
    x = composed_inputs(w, comp)
    d = to_device(x, w.io)
    got = run(d, x)
    del d
    torch.cuda.empty_cache()
    ref = oracle.forward_composed(x["q"], x["k"], x["v"], *(x[n] for n in WEIGHTS),
                                  x["gn_weight"], x["gn_bias"], x["depth_scale"],
                                  gn_eps=x["gn_eps"], w_head_pre=x["w_head_pre"],
                                  exact_mask=x["exact_mask"], w_kq_3d=x["w_kq_3d"])
    assert_every_element(got, ref, w.H, w.d, "longctx_4k " + comp)
