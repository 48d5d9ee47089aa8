"""The bounded-wait path of the fused kernels, exercised without a fault: a
kernel waits on a barrier nothing completes, gives up after a short budget,
and the host sees MTA_ERR_DEVICE_TIMEOUT; the context keeps working."""
import numpy as np
import pytest
import torch

import convolved_logit_attention_b200 as mta
from convolved_logit_attention_b200.workloads import Workload, make_inputs

pytestmark = pytest.mark.gpu


def test_expired_wait_is_reported_and_context_survives():
    from convolved_logit_attention_b200 import build
    build.build()
    mta.mta_sync_status()                      # clean start
    mta.mta_selftest_wait_timeout(1 << 20)     # ~0.5 ms of polling
    with pytest.raises(mta.MtaError) as exc:
        mta.mta_sync_status()
    assert exc.value.status == -6
    mta.mta_sync_status()                      # the flag was cleared
    w = Workload("after", 1, 2, 130, 64, 6, 11, 2, "bf16", seed=1)
    x = make_inputs(w)
    dev = torch.device("cuda", 0)
    d = {n: torch.from_numpy(x[n]).to(dev).to(torch.bfloat16) for n in ("q", "k", "v")}
    for n in ("w_kq", "w_head", "gn_weight", "gn_bias"):
        d[n] = torch.from_numpy(x[n]).to(dev)
    out = mta.mta_forward(d["q"], d["k"], d["v"], d["w_kq"], d["w_head"], d["gn_weight"],
                          d["gn_bias"], x["depth_scale"])
    mta.mta_sync_status()
    assert torch.isfinite(out.float()).all()


def _range_case(seed):
    w = Workload("range", 1, 2, 130, 64, 6, 11, 2, "bf16", seed=seed)
    x = make_inputs(w)
    dev = torch.device("cuda", 0)
    d = {n: torch.from_numpy(x[n]).to(dev).to(torch.bfloat16) for n in ("q", "k", "v")}
    for n in ("w_kq", "w_head", "gn_weight", "gn_bias"):
        d[n] = torch.from_numpy(x[n]).to(dev)
    shape = mta.shape_of(d["q"], d["w_kq"], d["w_head"])
    assert mta.mta_forward_path(shape) == mta.MTA_PATH_FUSED_TC
    return x, d


@pytest.mark.parametrize("which,value", [("q", 1.0e5), ("k", 1.0e6), ("q", -2.0e6)])
def test_values_beyond_fp16_range_stay_finite_and_are_flagged(which, value):
    # bf16 holds these, fp16 does not.  The prologue scales the query block
    # (or the folded-key block) that holds them by a power of two, so the
    # fused output stays finite; the call is flagged MTA_ERR_RANGE because the
    # fp16 future terms that the band correction cancels are then far too big
    # for the fused path's accuracy, and the materialised fp32 path, which
    # such inputs need, matches the oracle.
    import oracle
    x, d = _range_case(2)
    x[which] = x[which].copy()
    x[which][0, 1, 17, 3] = value           # exactly representable in bf16
    d[which][0, 1, 17, 3] = value
    mta.mta_sync_status()
    out = mta.mta_forward(d["q"], d["k"], d["v"], d["w_kq"], d["w_head"], d["gn_weight"],
                          d["gn_bias"], x["depth_scale"])
    with pytest.raises(mta.MtaError) as exc:
        mta.mta_sync_status()
    assert exc.value.status == -7
    assert torch.isfinite(out.float()).all()
    ref = oracle.forward(x["q"], x["k"], x["v"], x["w_kq"], x["w_head"], x["gn_weight"],
                         x["gn_bias"], x["depth_scale"])
    unf = mta.mta_forward_unfused(d["q"], d["k"], d["v"], d["w_kq"], d["w_head"],
                                  d["gn_weight"], d["gn_bias"], x["depth_scale"], check=True)
    got = unf.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    assert err.max() <= 2e-2 and np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 5e-3


def test_ordinary_inputs_raise_no_flag():
    x, d = _range_case(5)
    mta.mta_sync_status()
    mta.mta_forward(d["q"], d["k"], d["v"], d["w_kq"], d["w_head"], d["gn_weight"],
                    d["gn_bias"], x["depth_scale"], check=True)


def test_non_finite_input_is_reported():
    # an infinite query: the prologue cannot scale it into fp16 and raises the
    # range flag, which mta_sync_status reports (and clears)
    x, d = _range_case(3)
    d["q"][0, 1, 17, 3] = float("inf")
    mta.mta_sync_status()
    mta.mta_forward(d["q"], d["k"], d["v"], d["w_kq"], d["w_head"], d["gn_weight"],
                    d["gn_bias"], x["depth_scale"])
    with pytest.raises(mta.MtaError) as exc:
        mta.mta_sync_status()
    assert exc.value.status == -7
    mta.mta_sync_status()   # cleared


def test_check_flag_raises_at_the_call():
    # check=True synchronises the call's stream and raises what the device
    # flagged, so a torch caller does not get non-finite output silently
    x, d = _range_case(4)
    mta.mta_sync_status()
    out = mta.mta_forward(d["q"], d["k"], d["v"], d["w_kq"], d["w_head"], d["gn_weight"],
                          d["gn_bias"], x["depth_scale"], check=True)
    assert torch.isfinite(out.float()).all()
    d["k"][0, 0, 40, 5] = float("nan")
    with pytest.raises(mta.MtaError) as exc:
        mta.mta_forward(d["q"], d["k"], d["v"], d["w_kq"], d["w_head"], d["gn_weight"],
                        d["gn_bias"], x["depth_scale"], check=True)
    assert exc.value.status == -7
    mta.mta_sync_status()   # cleared
