"""Every element of every full-size workload against the fp64 oracle.

The benchmark's call (mta_forward, through the C ABI, in the launch
configuration bench.py times) on the T = 2048, 4096 and the six T = 16384
workloads, compared element by element with the oracle's full forward on the
same rounded inputs.  The fused kernel handles the two masks of "Multi-Token
Attention -- Paper Graph", section 3.4, Eq. (5) with a correction on the
tiles next to the diagonal and pairs query blocks; a mistake confined to one
class of rows (a band tile, a pair boundary, the ragged tail) would show up
here wherever it sits, and the failure message names the worst row.
"""
import numpy as np
import pytest
import torch

import oracle
import convolved_logit_attention_b200 as mta
from convolved_logit_attention_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TOL_BF16_MAXABS = 2e-2
TOL_BF16_RELL2 = 5e-3

FULL = ["pretrain_2k", "longctx_4k"] + sorted(n for n in WORKLOADS if n.startswith("long16k"))


@pytest.fixture(scope="module", autouse=True)
def _built():
    from convolved_logit_attention_b200 import build
    build.build()
    assert torch.cuda.is_available()


def _device(x, names=("q", "k", "v")):
    dev = torch.device("cuda", 0)
    d = {n: torch.from_numpy(np.ascontiguousarray(x[n])).to(dev).to(torch.bfloat16) for n in names}
    for n in ("w_kq", "w_head", "gn_weight", "gn_bias"):
        d[n] = torch.from_numpy(np.ascontiguousarray(x[n])).to(dev)
    return d


def assert_every_element(got, ref, H, d, what):
    """max-abs and rel-L2 over the whole output; on failure, where the worst
    element sits: batch entry, query row, head and channel."""
    assert np.isfinite(got).all(), what + ": non-finite output"
    err = np.abs(got - ref)
    maxabs = float(err.max())
    rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    b, t, c = np.unravel_index(int(err.argmax()), err.shape)
    row_err = err.max(axis=-1)                       # [B, T]
    bad_rows = int((row_err > TOL_BF16_MAXABS).sum())
    where = "worst at b=%d row=%d head=%d e=%d (row mod 128 = %d); %d rows over tolerance" % (
        b, t, c // d, c % d, t % 128, bad_rows)
    assert maxabs <= TOL_BF16_MAXABS and rel <= TOL_BF16_RELL2, \
        "%s: max-abs %.3g rel-L2 %.3g, %s" % (what, maxabs, rel, where)
    print("%s: max-abs %.4g rel-L2 %.4g over %d elements" % (what, maxabs, rel, got.size))
    return maxabs, rel


@pytest.mark.parametrize("name", FULL)
def test_full_size_every_element(name):
    w = WORKLOADS[name]
    x = make_inputs(w)
    d = _device(x)
    shape = mta.shape_of(d["q"], d["w_kq"], d["w_head"], x["gn_eps"])
    assert mta.mta_forward_path(shape) == mta.MTA_PATH_FUSED_TC
    out = mta.mta_forward(d["q"], d["k"], d["v"], d["w_kq"], d["w_head"], d["gn_weight"],
                          d["gn_bias"], x["depth_scale"], gn_eps=x["gn_eps"])
    mta.mta_sync_status()
    got = out.float().cpu().numpy().astype(np.float64)
    del d, out
    torch.cuda.empty_cache()
    ref = oracle.forward(x["q"], x["k"], x["v"], x["w_kq"], x["w_head"], x["gn_weight"],
                         x["gn_bias"], x["depth_scale"], gn_eps=x["gn_eps"])
    assert_every_element(got, ref, w.H, w.d, name)


GATE = np.array([-2.0, -0.5, 0.25, 1.5, 3.0, -1.0, 0.0, 0.75] * 4, dtype=np.float32)


def test_gated_output_full_size_every_element():
    """The T = 4096 workload with the sigmoid gate of "Group Normalization with
    Sigmoid Gating" in place of the depth scale, every element."""
    w = WORKLOADS["longctx_4k"]
    x = make_inputs(w)
    d = _device(x)
    gate = GATE[:w.H].copy()
    out = mta.mta_forward_gated(d["q"], d["k"], d["v"], d["w_kq"], d["w_head"], d["gn_weight"],
                                d["gn_bias"], torch.from_numpy(gate).cuda(), gn_eps=x["gn_eps"])
    mta.mta_sync_status()
    got = out.float().cpu().numpy().astype(np.float64)
    ref = oracle.forward(x["q"], x["k"], x["v"], x["w_kq"], x["w_head"], x["gn_weight"],
                         x["gn_bias"], 0.0, gn_eps=x["gn_eps"], gate=gate)
    assert_every_element(got, ref, w.H, w.d, "longctx_4k gated")


def test_materialised_path_full_size_every_element():
    """The materialised chain (mta_forward_unfused) on the T = 4096 workload,
    every element: its logits and A V run as tcgen05 tiles for bf16 I/O,
    with the fp32 maps of the chain in between."""
    w = WORKLOADS["longctx_4k"]
    x = make_inputs(w)
    d = _device(x)
    shape = mta.shape_of(d["q"], d["w_kq"], d["w_head"], x["gn_eps"])
    names = [mta.mta_kernel_name(shape, i, unfused=1) for i in range(4)]
    assert names == ["k_logits_tc", "k_conv", "k_softmax_mix", "k_pv_groupnorm_tc"]
    out = mta.mta_forward_unfused(d["q"], d["k"], d["v"], d["w_kq"], d["w_head"], d["gn_weight"],
                                  d["gn_bias"], x["depth_scale"], gn_eps=x["gn_eps"])
    mta.mta_sync_status()
    got = out.float().cpu().numpy().astype(np.float64)
    del d, out
    torch.cuda.empty_cache()
    ref = oracle.forward(x["q"], x["k"], x["v"], x["w_kq"], x["w_head"], x["gn_weight"],
                         x["gn_bias"], x["depth_scale"], gn_eps=x["gn_eps"])
    assert_every_element(got, ref, w.H, w.d, "longctx_4k materialised")
