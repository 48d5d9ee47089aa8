"""Pins of the oracle's compositions of the two MTA convolutions around the
softmax ("Multi-Token Attention -- Paper Graph", "Key-Query Convolution",
post-softmax variant and Eq. (4); "Head Mixing Convolution", pre-softmax
version; "Putting Everything Together: The Full MTA Module").

A composition runs, in this order, Mask_0, [key-query conv w_kq],
[head mix of the logits w_head_pre], Mask_-inf, softmax, [head mix w_head],
[key-query conv w_kq_post, Mask_0], [head mix w_head_post], A V, GroupNorm,
scale; a bracketed step with no weights is left out.  With exact_mask the
w_kq conv reads the unmasked logits under Eq. (4)'s indicator 1_{i >= j-j'}
instead of Mask_0's zeros.  The pins here do not come from the oracle: a brute force
built from scipy's true 2-D convolution and numpy on materialised maps, a
closed form for a single-tap kernel on the probabilities, reductions to
torch's causal attention, and invariants.
"""
import zlib

import numpy as np
import pytest
import scipy.signal
import scipy.special
import torch
import torch.nn.functional as F

import oracle
from tests.test_oracle_pins import rand_inputs


def true_conv2d(X, th):
    """[POST]/Eq. (4) index ranges: Y[b,h,i,j] = sum_{a,jj} th[h,a,jj]
    X[b,h,i-a, j-(jj-c_k//2)], zero outside the map.  scipy's 'full'
    convolution puts that sum at [i, j + c_k//2]."""
    B, H, T, _ = X.shape
    c_k = th.shape[-1]
    Y = np.empty_like(X)
    for b in range(B):
        for h in range(H):
            full = scipy.signal.convolve2d(X[b, h], th[h], mode="full")
            Y[b, h] = full[:T, c_k // 2: c_k // 2 + T]
    return Y


def indicator_conv(Afull, th):
    """Eq. (4) taken literally: C[b,h,i,j] = sum over taps (a, jj), with
    jp = jj - c_k//2, of th[h,a,jj] Afull[b,h,i-a,j-jp] where i-a >= 0,
    0 <= j-jp < T and j-jp <= i; Afull holds the unmasked logits."""
    B, H, T, _ = Afull.shape
    c_q, c_k = th.shape[1:]
    I = np.arange(T)[:, None]
    J = np.arange(T)[None, :]
    C = np.zeros_like(Afull)
    for a in range(c_q):
        for jj in range(c_k):
            r, c = I - a, J - (jj - c_k // 2)
            ok = (r >= 0) & (c >= 0) & (c < T) & (c <= I)
            shifted = Afull[:, :, np.clip(r, 0, T - 1), np.clip(c, 0, T - 1)]
            C += th[:, a, jj][None, :, None, None] * np.where(ok, shifted, 0.0)
    return C


def mix(Aw, w):
    B, H, T, _ = Aw.shape
    c_h = w.shape[-1]
    G = H // c_h
    return np.einsum("goi,bgitj->bgotj", w, Aw.reshape(B, G, c_h, T, T)).reshape(B, H, T, T)


def brute_force_composed(q, k, v, th, w, th_post, w_post, gw, gb, depth, gate=None, eps=1e-5,
                         w_pre=None, exact=False):
    B, H, T, d = q.shape
    causal = np.tril(np.ones((T, T), dtype=bool))
    Afull = np.einsum("bhie,bhje->bhij", q, k) / np.sqrt(d)
    A0 = np.where(causal, Afull, 0.0)
    if th is None:
        C = A0
    else:
        C = indicator_conv(Afull, th) if exact else true_conv2d(A0, th)
    if w_pre is not None:
        C = mix(C, w_pre)          # logits mixed before the second mask
    C = np.where(causal, C, -np.inf)
    P = scipy.special.softmax(C, axis=-1)
    A1 = mix(P, w) if w is not None else P
    A2 = np.where(causal, true_conv2d(A1, th_post), 0.0) if th_post is not None else A1
    A3 = mix(A2, w_post) if w_post is not None else A2
    O = A3 @ v
    Y = F.group_norm(torch.as_tensor(O).permute(0, 2, 1, 3).reshape(B * T, H * d), H,
                     torch.as_tensor(gw), torch.as_tensor(gb), eps).numpy().reshape(B, T, H, d)
    scale = (1.0 / (1.0 + np.exp(-gate)))[None, None, :, None] if gate is not None else depth
    return {"C": C, "P": P, "A1": A1, "A": A3, "O": O, "out": (scale * Y).reshape(B, T, H * d)}


# which of (w_kq, w_head, w_kq_post, w_head_post) a composition uses
COMPOSITIONS = {
    "repeat": (1, 1, 1, 1),
    "default": (1, 1, 0, 0),
    "post_kq_only": (0, 0, 1, 0),
    "both_post": (0, 0, 1, 1),
    "mix_then_post_kq": (0, 1, 1, 0),
    "pre_and_post_kq": (1, 0, 1, 0),
    "plain_attention": (0, 0, 0, 0),
}

SHAPES = [
    # B, H, T, d, c_q, c_k, c_h
    (1, 2, 9, 4, 3, 5, 2),
    (2, 4, 17, 8, 6, 11, 2),
    (1, 4, 13, 6, 2, 4, 4),      # even c_k
    (1, 3, 12, 5, 4, 3, 1),
    (1, 2, 7, 3, 1, 1, 2),       # 1x1 kernel
]


def composed_inputs(rng, shape, use):
    q, k, v, th, w, gw, gb = rand_inputs(rng, *shape)
    th_post = 0.5 * rng.standard_normal(th.shape)
    w_post = rng.standard_normal(w.shape)
    picked = [x if u else None for x, u in zip((th, w, th_post, w_post), use)]
    return q, k, v, picked, gw, gb


@pytest.mark.parametrize("name", sorted(COMPOSITIONS))
@pytest.mark.parametrize("shape", SHAPES)
def test_composition_matches_library_brute_force(shape, name):
    rng = np.random.default_rng(zlib.crc32(repr((shape, name)).encode()))
    q, k, v, ws, gw, gb = composed_inputs(rng, shape, COMPOSITIONS[name])
    gate = rng.standard_normal(shape[1]) if name == "repeat" else None
    ref = brute_force_composed(q, k, v, *ws, gw, gb, 0.7, gate=gate)
    out = oracle.forward_composed(q, k, v, *ws, gw, gb, 0.7, gate=gate)
    np.testing.assert_allclose(out, ref["out"], rtol=0, atol=1e-11)
    for b in range(shape[0]):
        st = oracle.stages_composed(q, k, v, *ws, gw, gb, 0.7, b=b, gate=gate)
        for key in ("P", "A1", "A", "O", "out"):
            want = ref[key][b] if key != "out" else ref["out"][b]
            np.testing.assert_allclose(st[key], want, rtol=0, atol=1e-11, err_msg=key)
        live = np.isfinite(ref["C"][b])
        assert np.array_equal(live, np.isfinite(st["C"]))
        np.testing.assert_allclose(st["C"][live], ref["C"][b][live], rtol=0, atol=1e-11)


@pytest.mark.parametrize("c_q,c_k", [(3, 5), (2, 4)])
def test_post_conv_single_tap_closed_form(c_q, c_k):
    # [POST] with one non-zero tap (i', j') shifts the probability map:
    # A[i][j] = P[i-i'][j-j'] when that entry lies inside the map, zero when
    # it does not, and zero for every future key j > i (Mask_0), even where
    # the shifted entry is a live probability.  P is the textbook causal
    # softmax, computed here with torch.
    rng = np.random.default_rng(20)
    H, T, d = 1, 12, 5
    q, k, v = (rng.standard_normal((1, H, T, d)) for _ in range(3))
    gw = np.ones(H * d); gb = np.zeros(H * d)
    logits = torch.as_tensor(q[0, 0] @ k[0, 0].T / np.sqrt(d))
    P = torch.softmax(logits.masked_fill(~torch.ones(T, T, dtype=torch.bool).tril(),
                                         float("-inf")), dim=-1).numpy()
    leaked = 0
    for ip in range(c_q):
        for jj in range(c_k):
            jp = jj - c_k // 2
            th = np.zeros((H, c_q, c_k)); th[0, ip, jj] = 1.0
            st = oracle.stages_composed(q, k, v, None, None, th, None, gw, gb, 1.0)
            A = st["A"][0]
            for i in range(T):
                for j in range(T):
                    r, c = i - ip, j - jp
                    inside = 0 <= r < T and 0 <= c < T
                    if j > i:
                        assert A[i, j] == 0.0
                        leaked += inside and P[r, c] > 0
                        continue
                    want = P[r, c] if inside else 0.0
                    assert abs(A[i, j] - want) < 1e-15, (ip, jp, i, j)
            np.testing.assert_allclose(st["O"][0], A @ v[0, 0], rtol=0, atol=1e-13)
    assert leaked > 0    # the case where Mask_0 after the conv matters did occur


def test_plain_composition_is_causal_attention():
    # With every convolution left out, the module is standard causal
    # softmax attention followed by the GroupNorm ("Standard Multi-Head
    # Attention"): compare with torch's SDPA and group_norm.
    rng = np.random.default_rng(21)
    B, H, T, d = 2, 4, 23, 8
    q, k, v = (rng.standard_normal((B, H, T, d)) for _ in range(3))
    gw = 1 + 0.1 * rng.standard_normal(H * d); gb = 0.1 * rng.standard_normal(H * d)
    O = F.scaled_dot_product_attention(*(torch.as_tensor(x) for x in (q, k, v)), is_causal=True)
    Y = F.group_norm(O.permute(0, 2, 1, 3).reshape(B * T, H * d), H, torch.as_tensor(gw),
                     torch.as_tensor(gb), 1e-5).reshape(B, T, H * d)
    out = oracle.forward_composed(q, k, v, None, None, None, None, gw, gb, 0.9)
    np.testing.assert_allclose(out, 0.9 * Y.numpy(), rtol=0, atol=1e-11)


def test_identity_repeat_reduces_to_default():
    # A repeated convolution with the identity kernels of "Practical Design
    # Choices" (theta_{0,0} = 1, w = I) leaves the default module unchanged.
    rng = np.random.default_rng(22)
    shape = (2, 4, 20, 8, 6, 11, 2)
    q, k, v, th, w, gw, gb = rand_inputs(rng, *shape)
    H, c_q, c_k, c_h = shape[1], shape[4], shape[5], shape[6]
    th_id = np.zeros((H, c_q, c_k)); th_id[:, 0, c_k // 2] = 1.0
    w_id = np.tile(np.eye(c_h), (H // c_h, 1, 1))
    out = oracle.forward_composed(q, k, v, th, w, th_id, w_id, gw, gb, 0.8)
    np.testing.assert_allclose(out, oracle.forward(q, k, v, th, w, gw, gb, 0.8), rtol=0,
                               atol=1e-13)


def test_zero_post_kernel_leaves_the_bias():
    # theta_post = 0 zeroes the attention that meets V, so every head output
    # is 0, its variance 0, and GroupNorm returns beta: out = scale * beta.
    rng = np.random.default_rng(23)
    B, H, T, d, c_q, c_k, c_h = 1, 4, 15, 6, 3, 5, 2
    q, k, v, th, w, gw, gb = rand_inputs(rng, B, H, T, d, c_q, c_k, c_h)
    out = oracle.forward_composed(q, k, v, th, w, np.zeros_like(th), w, gw, gb, 0.6)
    np.testing.assert_allclose(out, np.broadcast_to(0.6 * gb, out.shape), rtol=0, atol=1e-15)


def test_diff_mix_after_the_post_conv():
    # "Both post-softmax" with an identity key-query kernel and the DIFF
    # weights [1, -lambda] in the head mix gives SDPA(q1,k1,v1) -
    # lambda SDPA(q2,k2,v1) on the first head ("Head Mixing Convolution").
    rng = np.random.default_rng(24)
    B, H, T, d, lam = 1, 2, 19, 8, 0.45
    q, k, v = (rng.standard_normal((B, H, T, d)) for _ in range(3))
    th_id = np.zeros((H, 3, 5)); th_id[:, 0, 2] = 1.0
    w = np.array([[[1.0, -lam], [0.0, 1.0]]])
    st = oracle.stages_composed(q, k, v, None, None, th_id, w, np.ones(H * d), np.zeros(H * d), 1.0)
    tq, tk, tv = (torch.as_tensor(x[0]) for x in (q, k, v))
    a1 = F.scaled_dot_product_attention(tq[0:1], tk[0:1], tv[0:1], is_causal=True)[0]
    a2 = F.scaled_dot_product_attention(tq[1:2], tk[1:2], tv[0:1], is_causal=True)[0]
    np.testing.assert_allclose(st["O"][0], (a1 - lam * a2).numpy(), rtol=0, atol=1e-12)


def test_head_outputs_linear_in_post_kernel():
    # [POST] makes the attention, hence A V, linear in theta_post.
    rng = np.random.default_rng(25)
    B, H, T, d, c_q, c_k, c_h = 1, 2, 14, 6, 4, 5, 2
    q, k, v, th, w, gw, gb = rand_inputs(rng, B, H, T, d, c_q, c_k, c_h)
    t1, t2 = rng.standard_normal(th.shape), rng.standard_normal(th.shape)
    O = [oracle.stages_composed(q, k, v, th, w, tp, w, gw, gb, 1.0)["O"] for tp in (t1, t2, t1 + t2)]
    np.testing.assert_allclose(O[2], O[0] + O[1], rtol=0, atol=1e-12)


def test_repeat_causality():
    # Both masks of the repeat keep future tokens out of every output row.
    rng = np.random.default_rng(26)
    shape = (1, 4, 30, 8, 6, 11, 2)
    q, k, v, ws, gw, gb = composed_inputs(rng, shape, COMPOSITIONS["repeat"])
    out = oracle.forward_composed(q, k, v, *ws, gw, gb, 0.8)
    for t in (0, 4, 17, 28):
        q2, k2, v2 = q.copy(), k.copy(), v.copy()
        for x in (q2, k2, v2):
            x[:, :, t + 1:] += rng.standard_normal(x[:, :, t + 1:].shape)
        out2 = oracle.forward_composed(q2, k2, v2, *ws, gw, gb, 0.8)
        assert np.array_equal(out[:, : t + 1], out2[:, : t + 1])
        assert not np.allclose(out[:, t + 1:], out2[:, t + 1:])


@pytest.mark.parametrize("name", ["repeat", "post_kq_only", "both_post"])
def test_composed_rows_and_forward_agree(name):
    rng = np.random.default_rng(27)
    shape = (2, 4, 40, 8, 6, 11, 2)
    q, k, v, ws, gw, gb = composed_inputs(rng, shape, COMPOSITIONS[name])
    out = oracle.forward_composed(q, k, v, *ws, gw, gb, 0.8)
    idx = [0, 1, 4, 5, 6, 11, 20, 39]
    for b in range(shape[0]):
        r = oracle.rows_composed(q, k, v, *ws, gw, gb, 0.8, b, idx)
        np.testing.assert_allclose(r, out[b, idx], rtol=0, atol=1e-13)



# (w_kq, w_head_pre, w_head, w_kq_post, w_head_post, exact_mask)
PRE_COMPOSITIONS = {
    "both_pre": (1, 1, 0, 0, 0, 0),
    "logit_mix_only": (0, 1, 0, 0, 0, 0),
    "pre_mix_and_post_mix": (1, 1, 1, 0, 0, 0),
    "exact_default": (1, 0, 1, 0, 0, 1),
    "exact_both_pre": (1, 1, 0, 0, 0, 1),
    "exact_everything": (1, 1, 1, 1, 1, 1),
}


def pre_inputs(rng, shape, use):
    q, k, v, th, w, gw, gb = rand_inputs(rng, *shape)
    w_pre = rng.standard_normal(w.shape)
    th_post = 0.5 * rng.standard_normal(th.shape)
    w_post = rng.standard_normal(w.shape)
    picked = [x if u else None for x, u in zip((th, w_pre, w, th_post, w_post), use[:5])]
    return q, k, v, picked, bool(use[5]), gw, gb


def call_pre(fn, q, k, v, ws, exact, gw, gb, depth, **kw):
    th, w_pre, w, th_post, w_post = ws
    return fn(q, k, v, th, w, th_post, w_post, gw, gb, depth, w_head_pre=w_pre,
              exact_mask=exact, **kw)


@pytest.mark.parametrize("name", sorted(PRE_COMPOSITIONS))
@pytest.mark.parametrize("shape", SHAPES)
def test_pre_softmax_compositions_match_brute_force(shape, name):
    rng = np.random.default_rng(zlib.crc32(repr((shape, name, "pre")).encode()))
    q, k, v, ws, exact, gw, gb = pre_inputs(rng, shape, PRE_COMPOSITIONS[name])
    th, w_pre, w, th_post, w_post = ws
    ref = brute_force_composed(q, k, v, th, w, th_post, w_post, gw, gb, 0.7, w_pre=w_pre,
                               exact=exact)
    out = call_pre(oracle.forward_composed, q, k, v, ws, exact, gw, gb, 0.7)
    np.testing.assert_allclose(out, ref["out"], rtol=0, atol=1e-11)
    for b in range(shape[0]):
        st = call_pre(oracle.stages_composed, q, k, v, ws, exact, gw, gb, 0.7, b=b)
        for key in ("P", "A1", "A", "O"):
            np.testing.assert_allclose(st[key], ref[key][b], rtol=0, atol=1e-11, err_msg=key)
        live = np.isfinite(ref["C"][b])
        assert np.array_equal(live, np.isfinite(st["C"]))
        np.testing.assert_allclose(st["C"][live], ref["C"][b][live], rtol=0, atol=1e-11)


@pytest.mark.parametrize("c_q,c_k", [(3, 5), (4, 4)])
def test_exact_indicator_single_tap_closed_form(c_q, c_k):
    # Eq. (4) with one non-zero tap (i', j'): C[i][j] = q_{i-i'} . k_{j-j'} /
    # sqrt(d) when i-i' >= 0, 0 <= j-j' < T and j-j' <= i (the indicator), 0
    # otherwise, -inf for j > i.  Unlike Eq. (5)'s Mask_0 this keeps pairs
    # with i-i' < j-j' <= i, whose logits lie above the diagonal.
    rng = np.random.default_rng(40)
    H, T, d = 1, 13, 5
    q, k, v = (rng.standard_normal((1, H, T, d)) for _ in range(3))
    gw = np.ones(H * d); gb = np.zeros(H * d)
    kept_above = 0
    for ip in range(c_q):
        for jj in range(c_k):
            jp = jj - c_k // 2
            th = np.zeros((H, c_q, c_k)); th[0, ip, jj] = 1.0
            C = oracle.stages_composed(q, k, v, th, None, None, None, gw, gb, 1.0,
                                       exact_mask=True)["C"][0]
            for i in range(T):
                for j in range(T):
                    if j > i:
                        assert C[i, j] == -np.inf
                        continue
                    r, c = i - ip, j - jp
                    if r >= 0 and 0 <= c < T and c <= i:
                        want = float(q[0, 0, r] @ k[0, 0, c]) / np.sqrt(d)
                        kept_above += c > r
                    else:
                        want = 0.0
                    assert abs(C[i, j] - want) < 1e-12, (ip, jp, i, j)
    assert kept_above > 0


def test_exact_indicator_equals_two_pass_masking_for_one_query_tap():
    # With c_q = 1 the indicator 1_{i >= j-j'} and Mask_0 (j-j' <= i-0) agree.
    rng = np.random.default_rng(41)
    q, k, v, th, w, gw, gb = rand_inputs(rng, 2, 4, 23, 8, 1, 7, 2)
    a = oracle.forward_composed(q, k, v, th, w, None, None, gw, gb, 0.8)
    b = oracle.forward_composed(q, k, v, th, w, None, None, gw, gb, 0.8, exact_mask=True)
    assert np.array_equal(a, b)
    c = oracle.forward_composed(q, k, v, np.tile(th, (1, 3, 1)) / 3, w, None, None, gw, gb, 0.8,
                                exact_mask=True)
    assert not np.allclose(c, oracle.forward_composed(q, k, v, np.tile(th, (1, 3, 1)) / 3, w,
                                                      None, None, gw, gb, 0.8))


def test_logit_mix_is_softmax_of_mixed_logits():
    # "Head Mixing Convolution", pre-softmax version: with no key-query conv
    # the attention of head h is softmax(causal(sum_h' w[h][h'] q_h' k_h'^T /
    # sqrt(d))), computed here with torch.
    rng = np.random.default_rng(42)
    B, H, T, d, c_h = 1, 4, 19, 8, 2
    q, k, v = (rng.standard_normal((B, H, T, d)) for _ in range(3))
    w = rng.standard_normal((H // c_h, c_h, c_h))
    tq, tk = torch.as_tensor(q[0]), torch.as_tensor(k[0])
    logits = tq @ tk.transpose(-1, -2) / np.sqrt(d)                  # [H,T,T]
    mixed = torch.einsum("goi,gitj->gotj", torch.as_tensor(w),
                         logits.reshape(H // c_h, c_h, T, T)).reshape(H, T, T)
    P = torch.softmax(mixed.masked_fill(~torch.ones(T, T, dtype=torch.bool).tril(),
                                        float("-inf")), dim=-1)
    st = oracle.stages_composed(q, k, v, None, None, None, None, np.ones(H * d), np.zeros(H * d),
                                1.0, w_head_pre=w)
    np.testing.assert_allclose(st["P"], P.numpy(), rtol=0, atol=1e-13)
    np.testing.assert_allclose(st["O"], (P @ torch.as_tensor(v[0])).numpy(), rtol=0, atol=1e-12)


def test_exact_and_logit_mix_causality():
    rng = np.random.default_rng(43)
    shape = (1, 4, 28, 8, 6, 11, 2)
    q, k, v, ws, exact, gw, gb = pre_inputs(rng, shape, PRE_COMPOSITIONS["exact_everything"])
    out = call_pre(oracle.forward_composed, q, k, v, ws, exact, gw, gb, 0.8)
    for t in (0, 3, 16, 26):
        q2, k2, v2 = q.copy(), k.copy(), v.copy()
        for x in (q2, k2, v2):
            x[:, :, t + 1:] += rng.standard_normal(x[:, :, t + 1:].shape)
        out2 = call_pre(oracle.forward_composed, q2, k2, v2, ws, exact, gw, gb, 0.8)
        assert np.array_equal(out[:, : t + 1], out2[:, : t + 1])
        assert not np.allclose(out[:, t + 1:], out2[:, t + 1:])


@pytest.mark.parametrize("name", ["exact_everything", "both_pre"])
def test_pre_softmax_rows_and_forward_agree(name):
    rng = np.random.default_rng(44)
    shape = (2, 4, 40, 8, 6, 11, 2)
    q, k, v, ws, exact, gw, gb = pre_inputs(rng, shape, PRE_COMPOSITIONS[name])
    out = call_pre(oracle.forward_composed, q, k, v, ws, exact, gw, gb, 0.8)
    idx = [0, 1, 4, 5, 6, 11, 20, 39]
    for b in range(shape[0]):
        r = call_pre(oracle.rows_composed, q, k, v, ws, exact, gw, gb, 0.8, b=b, row_idx=idx)
        np.testing.assert_allclose(r, out[b, idx], rtol=0, atol=1e-13)


def conv3d_brute_force(q, k, v, th3, w, gw, gb, depth, exact=False, eps=1e-5):
    """ "Both pre-softmax (3D convolution view)": C^h = sum over the group's
    input heads h' of the 2-D conv (scipy, or the indicator form of Eq. (4))
    of head h''s logits with theta3[h][h'], then Mask_-inf, softmax, the
    post-softmax mix w (or none), A V, GroupNorm."""
    B, H, T, d = q.shape
    G, c_h = th3.shape[:2]
    causal = np.tril(np.ones((T, T), dtype=bool))
    Afull = np.einsum("bhie,bhje->bhij", q, k) / np.sqrt(d)
    A0 = np.where(causal, Afull, 0.0)
    C = np.zeros_like(Afull)
    for g in range(G):
        for ho in range(c_h):
            for hi in range(c_h):
                src = slice(g * c_h + hi, g * c_h + hi + 1)
                kern = th3[g, ho, hi][None]
                part = indicator_conv(Afull[:, src], kern) if exact else true_conv2d(A0[:, src], kern)
                C[:, g * c_h + ho] += part[:, 0]
    C = np.where(causal, C, -np.inf)
    P = scipy.special.softmax(C, axis=-1)
    A = mix(P, w) if w is not None else P
    O = A @ v
    Y = F.group_norm(torch.as_tensor(O).permute(0, 2, 1, 3).reshape(B * T, H * d), H,
                     torch.as_tensor(gw), torch.as_tensor(gb), eps).numpy().reshape(B, T, H * d)
    return {"C": C, "P": P, "A": A, "O": O, "out": depth * Y}


@pytest.mark.parametrize("exact", [False, True])
@pytest.mark.parametrize("shape", SHAPES)
def test_conv3d_matches_brute_force(shape, exact):
    rng = np.random.default_rng(zlib.crc32(repr((shape, exact, "3d")).encode()))
    B, H, T, d, c_q, c_k, c_h = shape
    q, k, v, _, w, gw, gb = rand_inputs(rng, *shape)
    th3 = 0.3 * rng.standard_normal((H // c_h, c_h, c_h, c_q, c_k))
    use_w = w if shape[1] != 3 else None       # with and without the post-softmax mix
    ref = conv3d_brute_force(q, k, v, th3, use_w, gw, gb, 0.7, exact=exact)
    out = oracle.forward_composed(q, k, v, None, use_w, None, None, gw, gb, 0.7, w_kq_3d=th3,
                                  exact_mask=exact)
    np.testing.assert_allclose(out, ref["out"], rtol=0, atol=1e-11)
    st = oracle.stages_composed(q, k, v, None, use_w, None, None, gw, gb, 0.7, b=0, w_kq_3d=th3,
                                exact_mask=exact)
    live = np.isfinite(ref["C"][0])
    assert np.array_equal(live, np.isfinite(st["C"]))
    np.testing.assert_allclose(st["C"][live], ref["C"][0][live], rtol=0, atol=1e-11)
    np.testing.assert_allclose(st["O"], ref["O"][0], rtol=0, atol=1e-11)


def test_conv3d_single_cross_head_tap():
    # A 3-D kernel whose one non-zero tap is theta3[out 0][in 1][i'][j'] = 1:
    # head 0's logits are head 1's masked logits shifted by (i', j') (Mask_0
    # zeros, not -inf, where that pair is not causal), and head 1's live
    # logits are all zero, so its attention is uniform over j <= i.
    rng = np.random.default_rng(50)
    H, T, d, c_q, c_k = 2, 12, 5, 3, 5
    q, k, v = (rng.standard_normal((1, H, T, d)) for _ in range(3))
    gw, gb = np.ones(H * d), np.zeros(H * d)
    for ip, jj in ((0, 2), (2, 0), (1, 4)):
        jp = jj - c_k // 2
        th3 = np.zeros((1, 2, 2, c_q, c_k)); th3[0, 0, 1, ip, jj] = 1.0
        st = oracle.stages_composed(q, k, v, None, None, None, None, gw, gb, 1.0, w_kq_3d=th3)
        for i in range(T):
            for j in range(i + 1):
                r, c = i - ip, j - jp
                want = float(q[0, 1, r] @ k[0, 1, c]) / np.sqrt(d) if (0 <= r and 0 <= c <= r) \
                    else 0.0
                assert abs(st["C"][0, i, j] - want) < 1e-12, (ip, jp, i, j)
                assert st["C"][1, i, j] == 0.0
            np.testing.assert_allclose(st["P"][1, i, : i + 1], 1.0 / (i + 1), rtol=0, atol=1e-15)


@pytest.mark.parametrize("exact", [False, True])
def test_separable_conv3d_is_conv_then_logit_mix(exact):
    # theta3[h][h'] = w_pre[h][h'] theta_{h'} makes the 3-D conv the key-query
    # conv followed by the pre-softmax head mix (the factorisation of the
    # 3-D view); a block-diagonal theta3 is the plain key-query conv.
    rng = np.random.default_rng(51)
    shape = (2, 4, 21, 8, 4, 5, 2)
    B, H, T, d, c_q, c_k, c_h = shape
    q, k, v, th, w, gw, gb = rand_inputs(rng, *shape)
    w_pre = rng.standard_normal(w.shape)
    G = H // c_h
    th3 = np.einsum("goi,gicd->goicd", w_pre, th.reshape(G, c_h, c_q, c_k))
    a = oracle.forward_composed(q, k, v, None, w, None, None, gw, gb, 0.8, w_kq_3d=th3,
                                exact_mask=exact)
    b = oracle.forward_composed(q, k, v, th, w, None, None, gw, gb, 0.8, w_head_pre=w_pre,
                                exact_mask=exact)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
    diag = np.einsum("oi,gicd->goicd", np.eye(c_h), th.reshape(G, c_h, c_q, c_k))
    c = oracle.forward_composed(q, k, v, None, w, None, None, gw, gb, 0.8, w_kq_3d=diag,
                                exact_mask=exact)
    e = oracle.forward_composed(q, k, v, th, w, None, None, gw, gb, 0.8, exact_mask=exact)
    np.testing.assert_allclose(c, e, rtol=0, atol=1e-13)
    with pytest.raises(RuntimeError):
        oracle.forward_composed(q, k, v, th, w, None, None, gw, gb, 0.8, w_kq_3d=th3)
