"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/mta.h declares, and rejects bad arguments before it
touches the device."""
import ctypes
import os
import re

import pytest

import convolved_logit_attention_b200 as mta
from convolved_logit_attention_b200 import _binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from convolved_logit_attention_b200 import build
    build.build()
    return mta.lib()


def header_functions():
    text = open(os.path.join(ROOT, "include", "mta.h")).read()
    return sorted(set(re.findall(r"MTA_API\s+[\w\s\*]*?\b(mta_\w+)\s*\(", text)))


def test_header_and_binding_agree():
    assert header_functions() == sorted(_binding.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    for name in header_functions():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_version_and_status_strings(L):
    assert mta.mta_version() == 100
    for code in _binding.STATUS:
        assert mta.mta_status_string(code)
    assert mta.mta_status_string(123) == "unknown status"


GOOD = dict(B=2, H=4, T=64, d=32, c_q=6, c_k=11, c_h=2)


def shape(**kw):
    args = dict(GOOD)
    args.update(kw)
    io = args.pop("io", "bf16")
    return mta.make_shape(io=io, **args)


@pytest.mark.parametrize("kw,status", [
    (dict(B=0), -1), (dict(T=0), -1), (dict(H=3), -1), (dict(c_q=0), -1),
    (dict(d=12), -2), (dict(d=136), -2), (dict(c_q=9), -2), (dict(c_k=16), -2),
    (dict(H=6, c_h=3), -2),
])
def test_forward_rejects_bad_shapes_before_launch(L, kw, status):
    s = shape(**kw)
    p = ctypes.c_void_p(1 << 20)    # aligned fake pointers: the call must not launch
    rc = L.mta_forward(ctypes.byref(s), p, p, p, p, p, p, p, 0.8, p, p, 1 << 40, None)
    assert rc == status
    assert mta.mta_workspace_size(s) == 0


def test_forward_rejects_null_misaligned_and_small_workspace(L):
    s = shape()
    a = ctypes.c_void_p(1 << 20)
    z = ctypes.c_void_p(0)
    bad = ctypes.c_void_p((1 << 20) + 4)
    need = mta.mta_workspace_size(s)
    assert need > 0
    args = [a] * 7
    assert L.mta_forward(ctypes.byref(s), z, *args[1:], 0.8, a, a, need, None) == -1
    assert L.mta_forward(ctypes.byref(s), bad, *args[1:], 0.8, a, a, need, None) == -3
    assert L.mta_forward(ctypes.byref(s), *args, 0.8, a, ctypes.c_void_p((1 << 20) + 16),
                         need, None) == -3
    assert L.mta_forward(ctypes.byref(s), *args, 0.8, a, a, need - 1, None) == -4
    assert L.mta_forward(ctypes.byref(s), *args, 0.8, a, z, need, None) == -1
    assert L.mta_forward_unfused(ctypes.byref(s), *args, 0.8, a, a,
                                 mta.mta_unfused_workspace_size(s) - 1, None) == -4


def test_gated_forward_argument_checks(L):
    # the gate is required and 4-byte aligned; the other checks are mta_forward's
    s = shape()
    a = ctypes.c_void_p(1 << 20)
    z = ctypes.c_void_p(0)
    need = mta.mta_workspace_size(s)
    args = [a] * 7
    assert L.mta_forward_gated(ctypes.byref(s), *args, z, a, a, need, None) == -1
    assert L.mta_forward_gated(ctypes.byref(s), *args, ctypes.c_void_p((1 << 20) + 2), a, a,
                               need, None) == -3
    assert L.mta_forward_gated(ctypes.byref(s), *args, a, a, a, need - 1, None) == -4
    bad = shape(c_h=3)
    assert L.mta_forward_gated(ctypes.byref(bad), *args, a, a, a, 1 << 40, None) == -1


def test_debug_attention_argument_checks(L):
    s = shape()
    a = ctypes.c_void_p(1 << 20)
    ws = mta.mta_unfused_workspace_size(s)
    assert L.mta_debug_attention(ctypes.byref(s), a, a, a, a, a, 2, a, ws, None) == -1
    big = shape(T=4096)
    assert L.mta_debug_attention(ctypes.byref(big), a, a, a, a, a, 0, a, 1 << 60, None) == -2


def test_unfused_workspace_is_two_fp32_maps(L):
    s = shape()
    assert mta.mta_unfused_workspace_size(s) == 2 * 4 * 2 * 4 * 64 * 64


@pytest.mark.parametrize("kw,path", [
    (dict(B=2, H=16, T=4096, d=128, c_q=6, c_k=11, c_h=2), 0),     # the benchmark workload
    (dict(B=1, H=16, T=16384, d=128, c_q=8, c_k=15, c_h=2), 0),
    (dict(B=8, H=4, T=256, d=64, c_q=4, c_k=15, c_h=2), 0),
    (dict(B=1, H=16, T=64, d=64, c_q=2, c_k=3, c_h=4), 0),
    (dict(B=1, H=16, T=16384, d=128, c_q=6, c_k=11, c_h=4), 0),    # split output heads
    (dict(B=1, H=16, T=256, d=128, c_q=6, c_k=11, c_h=8), 1),      # c_h * d > 512
    (dict(B=1, H=4, T=128, d=32, c_q=6, c_k=11, c_h=2), 1),        # d not 64 or 128
    (dict(B=1, H=4, T=128, d=32, c_q=6, c_k=11, c_h=2, io="f32"), 2),    # the fp32 workload
    (dict(B=1, H=4, T=128, d=128, c_q=6, c_k=11, c_h=2, io="f32"), 2),
    (dict(B=1, H=8, T=128, d=128, c_q=6, c_k=11, c_h=4, io="f32"), 1),   # c_h * d > 256
])
def test_forward_path_selection(L, kw, path):
    s = shape(**kw)
    assert mta.mta_forward_path(s) == path
    names = [mta.mta_kernel_name(s, i) for i in range(mta.mta_kernel_count(s))]
    if path == 0:   # prologue, main kernel, mix + GroupNorm
        assert names == ["k_fold", "k_mta_fused", "k_mix_groupnorm"]
    elif path == 2:  # one fused fp32 kernel, no workspace
        assert names == ["k_mta_fused_f32"]
        assert mta.mta_workspace_size(s) == 0
    else:           # the four materialised kernels; bf16 at d = 64 or 128 takes the
        # tensor-core logits and A V kernels
        tc = kw.get("io", "bf16") == "bf16" and kw["d"] in (64, 128)
        assert names == (["k_logits_tc", "k_conv", "k_softmax_mix", "k_pv_groupnorm_tc"] if tc
                         else ["k_logits", "k_conv", "k_softmax_mix", "k_pv_groupnorm"])


def test_backward_launch_names_follow_the_chain(L):
    # the recomputed logits take the chain's kernel; at d = 64 or 128 the fp32
    # products (A V, dV, dA = dO V^T, dQ, dK) are 3xTF32 tensor-core launches
    for kw, first, tf32 in ((dict(d=128), "k_logits_tc", True), (dict(d=32), "k_logits", False),
                            (dict(d=64, io="f32"), "k_logits", True)):
        names = mta.mta_backward_kernel_names(shape(**kw))
        assert len(names) == 14 and names[0] == first
        if tf32:
            assert [names[i] for i in (4, 6, 7, 11, 12)] == ["k_mm_tf32"] * 5
            assert "k_causal_mm" not in names
        else:
            assert names[7] == "k_logits" and names.count("k_causal_mm") == 4


def test_selftest_rejects_bad_budget(L):
    assert L.mta_selftest_wait_timeout(0, None) == -1
    assert L.mta_selftest_wait_timeout(1 << 31, None) == -1


def test_composed_launch_sequences_and_workspace(L):
    # "Putting Everything Together": each composition's launch list on the
    # materialised chain, and the default one on mta_forward's path.
    a = 1 << 20
    C = _binding.MtaComposition
    s = shape()
    seqs = {
        (a, a, a, a): ["k_logits", "k_conv", "k_softmax_mix", "k_conv", "k_head_mix",
                       "k_pv_groupnorm"],
        (None, None, a, None): ["k_logits", "k_softmax_mix", "k_conv", "k_pv_groupnorm"],
        (None, None, a, a): ["k_logits", "k_softmax_mix", "k_conv", "k_head_mix",
                             "k_pv_groupnorm"],
        (None, None, None, None): ["k_logits", "k_softmax_mix", "k_pv_groupnorm"],
        (a, None, a, None): ["k_logits", "k_conv", "k_softmax_mix", "k_conv", "k_pv_groupnorm"],
        # the pre-softmax head mix of the logits and the exact indicator of Eq. (4)
        (a, None, None, None, a, 0): ["k_logits", "k_conv", "k_head_mix", "k_softmax_mix",
                                      "k_pv_groupnorm"],
        (a, a, a, a, a, 1): ["k_logits", "k_conv", "k_head_mix", "k_softmax_mix", "k_conv",
                             "k_head_mix", "k_pv_groupnorm"],
        (a, a, None, None, None, 1): ["k_logits", "k_conv", "k_softmax_mix", "k_pv_groupnorm"],
        # the 3-D kernel in place of the key-query kernel
        (None, a, None, None, None, 0, a): ["k_logits", "k_conv", "k_softmax_mix",
                                            "k_pv_groupnorm"],
    }
    for ptrs, names in seqs.items():
        comp = C(*ptrs)
        assert mta.mta_composed_kernel_names(s, comp) == names
        assert L.mta_composed_workspace_size(ctypes.byref(s), ctypes.byref(comp)) == \
            mta.mta_unfused_workspace_size(s)
    fused = shape(B=2, H=16, T=4096, d=128, c_q=6, c_k=11, c_h=2)
    default = C(a, a, None, None)
    assert mta.mta_composed_kernel_names(fused, default) == \
        [mta.mta_kernel_name(fused, i) for i in range(mta.mta_kernel_count(fused))]
    # the default weights under the exact indicator of Eq. (4) stay on the
    # fused path (only the prologue's correction table changes)
    assert mta.mta_composed_kernel_names(fused, C(a, a, None, None, None, 1)) == \
        ["k_fold", "k_mta_fused", "k_mix_groupnorm"]
    assert L.mta_composed_workspace_size(ctypes.byref(fused), ctypes.byref(default)) == \
        mta.mta_workspace_size(fused)
    assert L.mta_composed_workspace_size(ctypes.byref(fused), None) == 0
    assert L.mta_composed_kernel_name(ctypes.byref(s), ctypes.byref(C(a, a, a, a)), 6) is None
    # bf16 at d = 64: the same chain with the tensor-core logits and A V kernels
    s64 = shape(d=64)
    assert mta.mta_composed_kernel_names(s64, C(a, a, a, a)) == \
        ["k_logits_tc", "k_conv", "k_softmax_mix", "k_conv", "k_head_mix", "k_pv_groupnorm_tc"]
    assert mta.mta_composed_kernel_names(shape(d=64, io="f32"), C(a, a, a, a)) == \
        ["k_logits", "k_conv", "k_softmax_mix", "k_conv", "k_head_mix", "k_pv_groupnorm"]


def test_composed_argument_checks(L):
    s = shape()
    a = ctypes.c_void_p(1 << 20)
    z = ctypes.c_void_p(0)
    C = _binding.MtaComposition
    rep = C(1 << 20, 1 << 20, 1 << 20, 1 << 20)
    need = mta.mta_unfused_workspace_size(s)

    def call(sh, comp, gw=a, gate=z, ws=a, nbytes=need, q=a):
        return L.mta_forward_composed(ctypes.byref(sh), q, a, a,
                                      ctypes.byref(comp) if comp is not None else None, gw, a,
                                      0.8, gate, a, ws, nbytes, None)

    assert call(s, None) == -1
    assert call(s, rep, gw=z) == -1
    assert call(s, rep, q=z) == -1
    assert call(s, C(1 << 20, 1 << 20, (1 << 20) + 8, None)) == -3
    assert call(s, C(1 << 20, None, None, None, (1 << 20) + 4, 0)) == -3
    assert call(s, C(None, None, None, None, None, 0, (1 << 20) + 4)) == -3
    assert call(s, C(1 << 20, None, None, None, None, 0, 1 << 20)) == -1   # w_kq and w_kq_3d
    assert call(s, rep, gate=ctypes.c_void_p((1 << 20) + 2)) == -3
    assert call(s, rep, nbytes=need - 1) == -4
    assert call(s, rep, ws=z) == -1
    assert call(shape(H=3), rep) == -1
    assert call(shape(c_q=9), rep) == -2
    # the default composition keeps mta_forward's checks (its workspace size)
    fused = shape(B=2, H=16, T=4096, d=128, c_q=6, c_k=11, c_h=2)
    fneed = mta.mta_workspace_size(fused)
    assert call(fused, C(1 << 20, 1 << 20, None, None), nbytes=fneed - 1) == -4


def test_ctypes_structs_match_the_c_header_layout(tmp_path):
    # The binding's ctypes mirrors of mta_shape and mta_composition must have
    # the header's field offsets and sizes; a C program built against
    # include/mta.h prints them.
    import subprocess
    fields = {"mta_shape": [f[0] for f in _binding.MtaShape._fields_],
              "mta_composition": [f[0] for f in _binding.MtaComposition._fields_]}
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "mta.h"', 'int main(void) {']
    for st, names in fields.items():
        lines.append('printf("%s size %%zu\\n", sizeof(%s));' % (st, st))
        for n in names:
            lines.append('printf("%s %s %%zu\\n", offsetof(%s, %s));' % (st, n, st, n))
    lines.append('return 0; }')
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)],
                   check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    got = {tuple(l.split()[:2]): int(l.split()[2]) for l in out if l.strip()}
    for st, cls in (("mta_shape", _binding.MtaShape), ("mta_composition", _binding.MtaComposition)):
        assert got[(st, "size")] == ctypes.sizeof(cls), st
        for n in fields[st]:
            assert got[(st, n)] == getattr(cls, n).offset, (st, n)
