"""Host-side arithmetic of bench.py: the FLOP counts of the compositions, the
work each kernel launch is credited with, and the roofline fraction."""
import bench
from convolved_logit_attention_b200.workloads import COMPOSITIONS, WORKLOADS

W = WORKLOADS["longctx_4k"]
LIVE = W.B * W.H * W.live_logits()


def test_composition_flops_add_one_term_per_step():
    # per live logit: 4d (QK^T and PV) + 2 c_q c_k per 2-D key-query conv
    # (2 c_h c_q c_k for the 3-D one) + 2 c_h per head mix
    conv, mix = 2 * W.c_q * W.c_k, 2 * W.c_h
    want = {
        "default": 4 * W.d + conv + mix,
        "repeat": 4 * W.d + 2 * conv + 2 * mix,
        "both_pre": 4 * W.d + conv + mix,
        "plain_attention": 4 * W.d,
        "logit_mix": 4 * W.d + mix,
        "conv3d": 4 * W.d + W.c_h * conv,
        "conv3d_exact_mix": 4 * W.d + W.c_h * conv + mix,
        "exact": 4 * W.d + conv + mix,
    }
    for name, per_logit in want.items():
        assert W.composition_flops(COMPOSITIONS[name]) == LIVE * per_logit, name
    assert W.composition_flops(COMPOSITIONS["default"]) == W.algorithmic_flops()


def test_conv_launches_are_credited_with_their_input_heads():
    two_d = LIVE * 2 * W.c_q * W.c_k
    for name, heads in (("default", 1), ("repeat", 1), ("conv3d", W.c_h), ("post_kq", 1)):
        comp = dict(COMPOSITIONS[name], c_h=W.c_h)
        bound, amount, unit = bench.kernel_units("k_conv", W, comp)
        assert (bound, unit) == ("alu", "FLOP")
        assert amount == two_d * heads, name
    # without a composition (the default entry points) a conv launch is 2-D
    assert bench.kernel_units("k_conv", W)[1] == two_d


def test_roofline_fraction_is_achieved_over_peak():
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1400.0}
    rl = bench.roofline("k_mta_fused", W, 0.5, peaks, "test")
    assert rl["bound"] == "tensor" and rl["unit"] == "TFLOP/s"
    assert abs(rl["achieved"] - W.algorithmic_flops() / 0.5e-3 / 1e12) < 1e-9
    assert abs(rl["frac"] - rl["achieved"] / 1500.0) < 1e-12
    hb = bench.roofline("k_head_mix", W, 0.25, peaks, "test")
    assert hb["bound"] == "hbm" and abs(hb["achieved"] - LIVE * 8 / 0.25e-3 / 1e9) < 1e-9
