"""Pins of the backward oracle (oracle/backward.py): gradients of the
forward the pages define, for the backward row that no kernel implements
yet.

The torch restatement of the forward must equal the C oracle's forward (which
has its own pins); every gradient must equal central finite differences of
the C oracle's forward along random directions, which shares no code with
autograd; the gradients of the affine parameters have closed forms; and
gradients respect causality.
"""
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
