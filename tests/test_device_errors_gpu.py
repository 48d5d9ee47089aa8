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


def test_values_beyond_fp16_range_are_reported():
    # bf16 holds 1e5, fp16 does not: the fused path's folded operands would
    # overflow, which the prologue reports instead of producing infinities.
    w = Workload("range", 1, 2, 130, 64, 6, 11, 2, "bf16", seed=2)
    x = make_inputs(w)
    dev = torch.device("cuda", 0)
    d = {n: torch.from_numpy(x[n]).to(dev).to(torch.bfloat16) for n in ("q", "k", "v")}
    for n in ("w_kq", "w_head", "gn_weight", "gn_bias"):
        d[n] = torch.from_numpy(x[n]).to(dev)
    shape = mta.shape_of(d["q"], d["w_kq"], d["w_head"])
    assert mta.mta_forward_path(shape) == mta.MTA_PATH_FUSED_TC
    d["q"][0, 1, 17, 3] = 1.0e5
    mta.mta_forward(d["q"], d["k"], d["v"], d["w_kq"], d["w_head"], d["gn_weight"],
                    d["gn_bias"], x["depth_scale"])
    with pytest.raises(mta.MtaError) as exc:
        mta.mta_sync_status()
    assert exc.value.status == -7
    mta.mta_sync_status()   # cleared


def test_check_flag_raises_at_the_call():
    # check=True synchronises the call's stream and raises what the device
    # flagged, so a torch caller does not get non-finite output silently
    w = Workload("range_check", 1, 2, 130, 64, 6, 11, 2, "bf16", seed=3)
    x = make_inputs(w)
    dev = torch.device("cuda", 0)
    d = {n: torch.from_numpy(x[n]).to(dev).to(torch.bfloat16) for n in ("q", "k", "v")}
    for n in ("w_kq", "w_head", "gn_weight", "gn_bias"):
        d[n] = torch.from_numpy(x[n]).to(dev)
    mta.mta_sync_status()
    out = mta.mta_forward(d["q"], d["k"], d["v"], d["w_kq"], d["w_head"], d["gn_weight"],
                          d["gn_bias"], x["depth_scale"], check=True)
    assert torch.isfinite(out.float()).all()
    d["k"][0, 0, 40, 5] = 2.0e5
    with pytest.raises(mta.MtaError) as exc:
        mta.mta_forward(d["q"], d["k"], d["v"], d["w_kq"], d["w_head"], d["gn_weight"],
                        d["gn_bias"], x["depth_scale"], check=True)
    assert exc.value.status == -7
    mta.mta_sync_status()   # cleared
