"""Pins of the backward oracle (oracle/backward.py): gradients of the
forward the pages define, for the backward row that no kernel implements
yet.

The torch restatement of the forward must equal the C oracle's forward (which
has its own pins); every gradient must equal central finite differences of
the C oracle's forward along random directions, which shares no code with
autograd; the gradients of the affine parameters have closed forms; and
gradients respect causality.
"""
import sys

import numpy as np
import pytest
import torch

import oracle
from oracle import backward
from tests.test_oracle_pins import rand_inputs

SHAPES = [
    # B, H, T, d, c_q, c_k, c_h
    (1, 2, 9, 4, 3, 5, 2),
    (2, 4, 12, 6, 4, 3, 2),
    (1, 4, 10, 5, 2, 4, 4),      # even c_k
]


def inputs_of(shape, seed):
    rng = np.random.default_rng(seed)
    q, k, v, th, w, gw, gb = rand_inputs(rng, *shape)
    return dict(zip(backward.NAMES, (q, k, v, th, w, gw, gb))), rng


@pytest.mark.parametrize("shape", SHAPES)
def test_torch_restatement_equals_the_c_oracle(shape):
    x, _ = inputs_of(shape, 60)
    ref = oracle.forward(*(x[n] for n in backward.NAMES), 0.7)
    got = backward.forward(*(torch.as_tensor(x[n]) for n in backward.NAMES), 0.7).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("shape", [(1, 2, 1, 4, 6, 11, 2), (2, 2, 2, 3, 8, 15, 1),
                                   (1, 4, 3, 4, 4, 3, 4)])
def test_shorter_than_the_kernel(shape):
    # T below c_q or c_k: every shift past the map reads zeros, as in the C
    # oracle; the restatement and its gradients stay defined
    x, rng = inputs_of(shape, 68)
    ref = oracle.forward(*(x[n] for n in backward.NAMES), 0.7)
    got = backward.forward(*(torch.as_tensor(x[n]) for n in backward.NAMES), 0.7).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    g = backward.gradients(x, rng.standard_normal(ref.shape), 0.7)
    assert all(np.isfinite(v).all() for v in g.values())


@pytest.mark.parametrize("shape", SHAPES)
def test_gradients_match_finite_differences_of_the_c_oracle(shape):
    # <grad_X, delta> = (f(X + h delta) - f(X - h delta)) . dout / (2 h),
    # with f the C oracle's forward; the truncation error is O(h^2).
    x, rng = inputs_of(shape, 61)
    dout = rng.standard_normal(oracle.forward(*(x[n] for n in backward.NAMES), 0.7).shape)
    g = backward.gradients(x, dout, 0.7)
    h = 1e-5
    for name in backward.NAMES:
        delta = rng.standard_normal(x[name].shape)
        plus, minus = dict(x), dict(x)
        plus[name] = x[name] + h * delta
        minus[name] = x[name] - h * delta
        fp = oracle.forward(*(plus[n] for n in backward.NAMES), 0.7)
        fm = oracle.forward(*(minus[n] for n in backward.NAMES), 0.7)
        fd = float(np.sum((fp - fm) * dout)) / (2 * h)
        an = float(np.sum(g[name] * delta))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_affine_parameter_gradients_closed_form():
    # out = s * (xhat * gamma + beta): d/dbeta = s * sum_t dout, and
    # d/dgamma = s * sum_t xhat * dout, with xhat = (out/s - beta) / gamma.
    shape = (2, 4, 11, 6, 3, 5, 2)
    x, rng = inputs_of(shape, 62)
    B, H, T, d = shape[:4]
    s = 0.7
    out = oracle.forward(*(x[n] for n in backward.NAMES), s)
    dout = rng.standard_normal(out.shape)
    g = backward.gradients(x, dout, s)
    np.testing.assert_allclose(g["gn_bias"], s * dout.sum(axis=(0, 1)), rtol=0, atol=1e-12)
    xhat = (out / s - x["gn_bias"]) / x["gn_weight"]
    np.testing.assert_allclose(g["gn_weight"], s * (xhat * dout).sum(axis=(0, 1)), rtol=0,
                               atol=1e-10)


def test_gradients_are_causal():
    # With dout zero on every row after t, no token after t receives a
    # gradient: row i reads queries i-c_q+1 .. i and keys and values <= i.
    shape = (1, 2, 14, 5, 4, 5, 2)
    x, rng = inputs_of(shape, 63)
    out = oracle.forward(*(x[n] for n in backward.NAMES), 0.7)
    for t in (3, 9):
        dout = rng.standard_normal(out.shape)
        dout[:, t + 1:] = 0.0
        g = backward.gradients(x, dout, 0.7)
        for name in ("q", "k", "v"):
            assert np.all(g[name][:, :, t + 1:] == 0.0), (name, t)
            assert np.abs(g[name][:, :, : t + 1]).max() > 0.0


GATE = np.array([-1.5, 0.25, 2.0, -0.5])


@pytest.mark.parametrize("shape", SHAPES)
def test_gated_restatement_and_gate_gradient(shape):
    # "Group Normalization with Sigmoid Gating": the torch restatement with a
    # gate equals the C oracle's gated forward, and every gradient (the
    # gate's included) equals central finite differences of that C forward.
    x, rng = inputs_of(shape, 65)
    H = shape[1]
    gate = GATE[:H].copy()
    c_fwd = lambda xx, gg: oracle.forward(*(xx[n] for n in backward.NAMES), 0.0, gate=gg)
    ref = c_fwd(x, gate)
    got = backward.forward(*(torch.as_tensor(x[n]) for n in backward.NAMES), 0.0,
                           gate=torch.as_tensor(gate)).numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
    dout = rng.standard_normal(ref.shape)
    g = backward.gradients(x, dout, 0.0, gate=gate)
    assert set(g) == set(backward.NAMES) | {"gate"}
    h = 1e-5
    for name in list(backward.NAMES) + ["gate"]:
        base = gate if name == "gate" else x[name]
        delta = rng.standard_normal(base.shape)
        if name == "gate":
            fp, fm = c_fwd(x, gate + h * delta), c_fwd(x, gate - h * delta)
        else:
            plus, minus = dict(x), dict(x)
            plus[name] = x[name] + h * delta
            minus[name] = x[name] - h * delta
            fp, fm = c_fwd(plus, gate), c_fwd(minus, gate)
        fd = float(np.sum((fp - fm) * dout)) / (2 * h)
        an = float(np.sum(g[name] * delta))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


ROW_SHAPES = [
    # B, H, T, d, c_q, c_k, c_h
    (2, 4, 23, 6, 6, 11, 2),
    (1, 4, 19, 5, 3, 4, 4),      # even c_k
    (1, 3, 17, 4, 8, 15, 1),
]


@pytest.mark.parametrize("shape", ROW_SHAPES)
def test_row_restricted_forward_equals_the_c_oracle_rows(shape):
    # forward_rows recomputes only what the chosen rows depend on; it must
    # give the C oracle's rows (computed there one row at a time from scratch),
    # with and without the gate.
    x, _ = inputs_of(shape, 66)
    B, H, T = shape[:3]
    rows = [0, 1, 2, 7, T // 2, T - 2, T - 1]
    ts = [torch.as_tensor(x[n]) for n in backward.NAMES]
    got = backward.forward_rows(*ts, 0.7, rows).numpy()
    gate = GATE[:H].copy()
    got_g = backward.forward_rows(*ts, 0.0, rows, gate=torch.as_tensor(gate)).numpy()
    for b in range(B):
        ref = oracle.rows(*(x[n] for n in backward.NAMES), 0.7, b, rows)
        np.testing.assert_allclose(got[b], ref, rtol=0, atol=1e-12)
        ref_g = oracle.rows(*(x[n] for n in backward.NAMES), 0.0, b, rows, gate=gate)
        np.testing.assert_allclose(got_g[b], ref_g, rtol=0, atol=1e-12)


@pytest.mark.parametrize("shape", ROW_SHAPES)
def test_row_restricted_gradients_equal_full_gradients(shape):
    # An upstream gradient that vanishes off a few rows: the gradients through
    # forward_rows equal those of the full restatement (which the finite
    # difference pins above tie to the C oracle).
    x, rng = inputs_of(shape, 67)
    B, H, T, d = shape[:4]
    rows = [1, 5, T - 1]
    dout = np.zeros((B, T, H * d))
    dout[:, rows] = rng.standard_normal((B, len(rows), H * d))
    full = backward.gradients(x, dout, 0.7)
    part = backward.gradients_rows(x, rows, dout[:, rows], 0.7)
    for n in backward.NAMES:
        np.testing.assert_allclose(part[n], full[n], rtol=0, atol=1e-11, err_msg=n)


# (w_kq, w_kq_3d, w_head_pre, w_head, w_kq_post, w_head_post, exact_mask)
COMPOSED = {
    "repeat": (1, 0, 0, 1, 1, 1, 0),
    "exact_both_pre": (1, 0, 1, 0, 0, 0, 1),
    "conv3d_exact_mix": (0, 1, 0, 1, 0, 0, 1),
}


def composed_inputs_of(shape, use, seed):
    rng = np.random.default_rng(seed)
    q, k, v, th, w, gw, gb = rand_inputs(rng, *shape)
    B, H, T, d, c_q, c_k, c_h = shape
    th3 = 0.3 * rng.standard_normal((H // c_h, c_h, c_h, c_q, c_k))
    extra = dict(w_kq=th, w_kq_3d=th3, w_head_pre=rng.standard_normal(w.shape), w_head=w,
                 w_kq_post=0.5 * rng.standard_normal(th.shape),
                 w_head_post=rng.standard_normal(w.shape))
    x = dict(q=q, k=k, v=v, gn_weight=gw, gn_bias=gb)
    for name, u in zip(("w_kq", "w_kq_3d", "w_head_pre", "w_head", "w_kq_post", "w_head_post"),
                       use[:6]):
        x[name] = extra[name] if u else None
    return x, bool(use[6]), rng


def c_forward(x, exact, depth=0.7):
    return oracle.forward_composed(x["q"], x["k"], x["v"], x["w_kq"], x["w_head"], x["w_kq_post"],
                                   x["w_head_post"], x["gn_weight"], x["gn_bias"], depth,
                                   w_head_pre=x["w_head_pre"], exact_mask=exact,
                                   w_kq_3d=x["w_kq_3d"])


@pytest.mark.parametrize("name", sorted(COMPOSED))
def test_composed_restatement_and_gradients(name):
    # The torch restatement of each composition equals the C oracle's
    # composed forward, and its autograd gradients equal central finite
    # differences of that C forward along random directions.
    shape = (1, 4, 10, 4, 3, 5, 2)
    x, exact, rng = composed_inputs_of(shape, COMPOSED[name], 64)
    ref = c_forward(x, exact)
    ts = {n: None if x.get(n) is None else torch.as_tensor(x[n]) for n in backward.COMPOSED_NAMES}
    np.testing.assert_allclose(backward.forward_composed(ts, 0.7, exact).numpy(), ref, rtol=0,
                               atol=1e-12)
    dout = rng.standard_normal(ref.shape)
    g = backward.gradients_composed(x, dout, 0.7, exact)
    h = 1e-5
    for n, grad in g.items():
        delta = rng.standard_normal(x[n].shape)
        plus, minus = dict(x), dict(x)
        plus[n] = x[n] + h * delta
        minus[n] = x[n] - h * delta
        fd = float(np.sum((c_forward(plus, exact) - c_forward(minus, exact)) * dout)) / (2 * h)
        an = float(np.sum(grad * delta))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, n, fd, an)


# Planted mistakes in the torch restatement; some pin above must catch each.
BACKWARD_MUTATIONS = [
    ("key shift sign", "C = C + w_kq[:, ip, jj].view(1, H, 1, 1) * _shift(A0, ip, jp)",
     "C = C + w_kq[:, ip, jj].view(1, H, 1, 1) * _shift(A0, ip, -jp)"),
    ("mix transposed", 'A = torch.einsum("goi,bgitj->bgotj", w_head,',
     'A = torch.einsum("gio,bgitj->bgotj", w_head,'),
    ("unbiased variance", "var = ((O - mean) ** 2).mean(dim=-1, keepdim=True)\n    xhat",
     "var = ((O - mean) ** 2).sum(dim=-1, keepdim=True) / (d - 1)\n    xhat"),
    ("exact indicator against the shifted query",
     "S = torch.where(J - jp <= I, S, torch.zeros((), dtype=X.dtype))",
     "S = torch.where(J - jp <= I - ip, S, torch.zeros((), dtype=X.dtype))"),
    ("post conv not masked", 'A = torch.where(causal, _conv(A, t["w_kq_post"], False), zero)',
     'A = _conv(A, t["w_kq_post"], False)'),
    ("gate not squashed", "return torch.sigmoid(gate).view(1, H, 1, 1)",
     "return gate.view(1, H, 1, 1)"),
    ("row restatement: key shift sign", "jp = jj - R                                # C[j]",
     "jp = R - jj                                # C[j]"),
    ("row restatement: no Mask_0", "keep = torch.arange(n) <= r                    # Mask_0",
     "keep = torch.arange(n) <= i                    # Mask_0"),
    ("row restatement: gate ignored",
     "scale = depth_scale if gate is None else torch.sigmoid(gate).view(1, H, 1)",
     "scale = depth_scale"),
]


@pytest.mark.parametrize("name,before,after", BACKWARD_MUTATIONS,
                         ids=[m[0] for m in BACKWARD_MUTATIONS])
def test_backward_pins_catch_planted_mistakes(monkeypatch, tmp_path, name, before, after):
    import importlib.util
    src = open(backward.__file__).read()
    assert src.count(before) == 1, before
    path = tmp_path / "mutant_backward.py"
    path.write_text(src.replace(before, after))
    spec = importlib.util.spec_from_file_location("mutant_backward", str(path))
    mutant = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mutant)
    monkeypatch.setattr(sys.modules[__name__], "backward", mutant)
    checks = [lambda: test_torch_restatement_equals_the_c_oracle(SHAPES[1]),
              lambda: test_gradients_match_finite_differences_of_the_c_oracle(SHAPES[1]),
              lambda: test_gated_restatement_and_gate_gradient(SHAPES[1]),
              lambda: test_row_restricted_forward_equals_the_c_oracle_rows(ROW_SHAPES[0])]
    checks += [lambda n=n: test_composed_restatement_and_gradients(n) for n in sorted(COMPOSED)]
    caught = 0
    for check in checks:
        try:
            check()
        except AssertionError:
            caught += 1
    assert caught, "no pin caught: " + name
