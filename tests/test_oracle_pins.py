"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test checks the oracle against one of: a library routine on a special
case (torch's causal scaled-dot-product attention, conv2d, softmax,
group_norm), a closed form read off the pages' equations, an invariant of the
definitions, or the receptive-field fixture under tests/golden/.

Page references are to "Multi-Token Attention -- Paper Graph", section 3.4,
unless stated otherwise.
"""
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_inputs(rng, B, H, T, d, c_q, c_k, c_h, kscale=0.3):
    q = rng.standard_normal((B, H, T, d))
    k = rng.standard_normal((B, H, T, d))
    v = rng.standard_normal((B, H, T, d))
    th = kscale * rng.standard_normal((H, c_q, c_k))
    w = rng.standard_normal((H // c_h, c_h, c_h))
    gw = 1.0 + 0.1 * rng.standard_normal(H * d)
    gb = 0.1 * rng.standard_normal(H * d)
    return q, k, v, th, w, gw, gb


def brute_force(q, k, v, th, w, gw, gb, depth, eps=1e-5):
    """The pages' forward composed from library routines on materialised
    T x T maps (tiny T only): masked logits, a true 2-D convolution done by
    torch's cross-correlation with the kernel flipped, softmax, einsum head
    mixing, matmul, torch group_norm with one group per head."""
    q, k, v, th, w, gw, gb = (torch.as_tensor(x, dtype=torch.float64)
                              for x in (q, k, v, th, w, gw, gb))
    B, H, T, d = q.shape
    _, c_q, c_k = th.shape
    c_h = w.shape[-1]
    G = H // c_h
    A = q @ k.transpose(-1, -2) / np.sqrt(d)                       # "Standard MHA"
    causal = torch.ones(T, T, dtype=torch.bool).tril()
    A0 = torch.where(causal, A, torch.zeros(()))                    # Mask_0, Eq. (5)
    # true convolution: C[i,j] = sum th[a,b] A0[i-a, j-(b-c_k//2)]; with the
    # kernel flipped both ways conv2d's correlation needs c_q-1 zero rows on
    # top and ceil(c_k/2)-1 / floor(c_k/2) zero columns left / right.
    X = F.pad(A0.reshape(B * H, 1, T, T),
              ((c_k + 1) // 2 - 1, c_k // 2, c_q - 1, 0))
    Cs = []
    for h in range(H):
        Wk = th[h].flip(0, 1).reshape(1, 1, c_q, c_k)
        Xh = X.reshape(B, H, 1, X.shape[-2], X.shape[-1])[:, h]
        Cs.append(F.conv2d(Xh, Wk)[:, 0])
    C = torch.stack(Cs, dim=1)                                      # [B,H,T,T]
    C = C.masked_fill(~causal, float("-inf"))                       # Mask_-inf
    P = torch.softmax(C, dim=-1)
    Pg = P.reshape(B, G, c_h, T, T)
    Amix = torch.einsum("goi,bgitj->bgotj", w, Pg).reshape(B, H, T, T)   # Eq. (7)
    O = Amix @ v                                                     # [B,H,T,d]
    Ocat = O.permute(0, 2, 1, 3).reshape(B * T, H * d)
    Y = F.group_norm(Ocat, H, gw, gb, eps).reshape(B, T, H * d)
    return {"C": C, "P": P, "A": Amix, "O": O, "out": depth * Y}


SHAPES = [
    # B, H, T, d, c_q, c_k, c_h
    (1, 2, 9, 4, 3, 5, 2),
    (2, 4, 17, 8, 6, 11, 2),
    (1, 4, 13, 6, 2, 4, 4),      # even c_k
    (1, 3, 12, 5, 4, 3, 1),      # no mixing partner
    (1, 4, 20, 8, 8, 15, 1),
    (1, 2, 7, 3, 1, 1, 2),       # 1x1 kernel
]


@pytest.mark.parametrize("shape", SHAPES)
def test_oracle_matches_library_composition(shape):
    rng = np.random.default_rng(hash(shape) % 2**32)
    q, k, v, th, w, gw, gb = rand_inputs(rng, *shape)
    ref = brute_force(q, k, v, th, w, gw, gb, 0.7)
    out = oracle.forward(q, k, v, th, w, gw, gb, 0.7)
    np.testing.assert_allclose(out, ref["out"].numpy(), rtol=0, atol=1e-11)
    for b in range(shape[0]):
        st = oracle.stages(q, k, v, th, w, gw, gb, 0.7, b=b)
        for key in ("P", "A", "O"):
            np.testing.assert_allclose(st[key], ref[key][b].numpy(), rtol=0, atol=1e-11)
        Cr = ref["C"][b].numpy()
        live = np.isfinite(Cr)
        assert np.array_equal(live, np.isfinite(st["C"]))
        np.testing.assert_allclose(st["C"][live], Cr[live], rtol=0, atol=1e-11)
        np.testing.assert_allclose(st["out"], ref["out"][b].numpy(), rtol=0, atol=1e-11)


def test_identity_kernels_give_causal_softmax_attention():
    # "Practical Design Choices": theta_{0,0} = 1 and w = I make MTA standard
    # attention; compare with torch's causal SDPA and group_norm.
    rng = np.random.default_rng(1)
    B, H, T, d, c_q, c_k, c_h = 2, 4, 33, 16, 6, 11, 2
    q, k, v, _, _, gw, gb = rand_inputs(rng, B, H, T, d, c_q, c_k, c_h)
    th = np.zeros((H, c_q, c_k)); th[:, 0, c_k // 2] = 1.0
    w = np.tile(np.eye(c_h), (H // c_h, 1, 1))
    tq, tk, tv = (torch.as_tensor(x) for x in (q, k, v))
    O = F.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    Y = F.group_norm(O.permute(0, 2, 1, 3).reshape(B * T, H * d), H,
                     torch.as_tensor(gw), torch.as_tensor(gb), 1e-5).reshape(B, T, H * d)
    out = oracle.forward(q, k, v, th, w, gw, gb, 0.8)
    np.testing.assert_allclose(out, 0.8 * Y.numpy(), rtol=0, atol=1e-11)
    st = oracle.stages(q, k, v, th, w, gw, gb, 0.8, b=1)
    np.testing.assert_allclose(st["O"], O[1].numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("c_q,c_k", [(6, 11), (3, 4), (2, 3)])
def test_single_tap_kernel_closed_form(c_q, c_k):
    # Eq. (4)/(5) with one non-zero tap (i', j'): C[i][j] is q_{i-i'} . k_{j-j'}
    # / sqrt(d) when that pair is causal and inside the sequence, zero when it
    # is not (Mask_0 gives zeros, not -inf), and -inf for j > i.
    rng = np.random.default_rng(2)
    H, T, d = 1, 14, 5
    q, k, v = (rng.standard_normal((1, H, T, d)) for _ in range(3))
    w = np.ones((1, 1, 1)); gw = np.ones(H * d); gb = np.zeros(H * d)
    for ip in range(c_q):
        for jj in range(c_k):
            jp = jj - c_k // 2
            th = np.zeros((H, c_q, c_k)); th[0, ip, jj] = 1.0
            C = oracle.stages(q, k, v, th, w, gw, gb, 1.0)["C"][0]
            for i in range(T):
                for j in range(T):
                    if j > i:
                        assert C[i, j] == -np.inf
                        continue
                    r, c = i - ip, j - jp
                    if 0 <= r < T and 0 <= c <= r:
                        want = float(q[0, 0, r] @ k[0, 0, c]) / np.sqrt(d)
                    else:
                        want = 0.0
                    assert abs(C[i, j] - want) < 1e-12, (ip, jp, i, j)


def test_receptive_field_matches_golden():
    # The set of (r - i, c - j) offsets read by C[i][j], found by probing each
    # tap alone, equals the fixture taken from the page's index ranges.
    rows = []
    with open(os.path.join(GOLDEN, "receptive_field.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(tuple(int(x) for x in line.split()))
    rng = np.random.default_rng(3)
    T, d = 24, 3
    q, k, v = (rng.standard_normal((1, 1, T, d)) for _ in range(3))
    logits = (q[0, 0] @ k[0, 0].T) / np.sqrt(d)
    w = np.ones((1, 1, 1)); gw = np.ones(d); gb = np.zeros(d)
    i, j = 23, 8    # every tap of the largest kernel stays causal and inside
    for c_q, c_k, qmin, qmax, kmin, kmax in rows:
        offs = set()
        for ip in range(c_q):
            for jj in range(c_k):
                th = np.zeros((1, c_q, c_k)); th[0, ip, jj] = 1.0
                val = oracle.stages(q, k, v, th, w, gw, gb, 1.0)["C"][0, i, j]
                hit = [(r - i, c - j) for r in range(T) for c in range(r + 1)
                       if abs(logits[r, c] - val) < 1e-13]
                assert len(hit) == 1
                offs.add(hit[0])
        dr = sorted({o[0] for o in offs}); dc = sorted({o[1] for o in offs})
        assert (dr[0], dr[-1], dc[0], dc[-1]) == (qmin, qmax, kmin, kmax)
        assert len(offs) == c_q * c_k


def test_zero_kernel_gives_prefix_mean():
    # theta = 0 makes every live logit 0, so the softmax is uniform over
    # j <= i and (with w = I) the head output is the mean of v_0..v_i.
    rng = np.random.default_rng(4)
    H, T, d, c_h = 2, 19, 7, 2
    q, k, v = (rng.standard_normal((1, H, T, d)) for _ in range(3))
    th = np.zeros((H, 3, 5)); w = np.eye(2)[None]
    st = oracle.stages(q, k, v, th, w, np.ones(H * d), np.zeros(H * d), 1.0)
    want = np.cumsum(v[0], axis=1) / np.arange(1, T + 1)[None, :, None]
    np.testing.assert_allclose(st["O"], want, rtol=0, atol=1e-13)
    for i in range(T):
        np.testing.assert_allclose(st["P"][:, i, : i + 1], 1.0 / (i + 1), rtol=0, atol=1e-15)


def test_diff_transformer_special_case():
    # "Head Mixing Convolution": DIFF Transformer is head mixing with c_h = 2
    # and weights [1, -lambda]; with identity kq kernels the first head's
    # output is SDPA(q1,k1,v1) - lambda SDPA(q2,k2,v1).
    rng = np.random.default_rng(5)
    B, H, T, d, lam = 1, 2, 21, 8, 0.37
    q, k, v = (rng.standard_normal((B, H, T, d)) for _ in range(3))
    th = np.zeros((H, 4, 7)); th[:, 0, 3] = 1.0
    w = np.array([[[1.0, -lam], [0.0, 1.0]]])
    st = oracle.stages(q, k, v, th, w, np.ones(H * d), np.zeros(H * d), 1.0)
    tq, tk, tv = (torch.as_tensor(x[0]) for x in (q, k, v))
    a1 = F.scaled_dot_product_attention(tq[0:1], tk[0:1], tv[0:1], is_causal=True)[0]
    a2 = F.scaled_dot_product_attention(tq[1:2], tk[1:2], tv[0:1], is_causal=True)[0]
    b2 = F.scaled_dot_product_attention(tq[1:2], tk[1:2], tv[1:2], is_causal=True)[0]
    np.testing.assert_allclose(st["O"][0], (a1 - lam * a2).numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(st["O"][1], b2.numpy(), rtol=0, atol=1e-12)


def test_causality_future_tokens_do_not_leak():
    # Eq. (5): the two masks keep future tokens out of every output row.
    rng = np.random.default_rng(6)
    B, H, T, d, c_q, c_k, c_h = 1, 4, 30, 8, 6, 11, 2
    q, k, v, th, w, gw, gb = rand_inputs(rng, B, H, T, d, c_q, c_k, c_h)
    out = oracle.forward(q, k, v, th, w, gw, gb, 0.8)
    for t in (0, 5, 17, 28):
        q2, k2, v2 = q.copy(), k.copy(), v.copy()
        q2[:, :, t + 1:] += rng.standard_normal(q2[:, :, t + 1:].shape)
        k2[:, :, t + 1:] += rng.standard_normal(k2[:, :, t + 1:].shape)
        v2[:, :, t + 1:] += rng.standard_normal(v2[:, :, t + 1:].shape)
        out2 = oracle.forward(q2, k2, v2, th, w, gw, gb, 0.8)
        assert np.array_equal(out[:, : t + 1], out2[:, : t + 1])
        assert not np.allclose(out[:, t + 1:], out2[:, t + 1:])


def test_row_sums_pre_and_post_mix():
    # Pre-mix rows are probability distributions over j <= i ("Standard MHA");
    # post-mix rows sum to sum_h' w[h][h'] (Eq. (7) is linear in the rows).
    rng = np.random.default_rng(7)
    B, H, T, d, c_q, c_k, c_h = 1, 4, 25, 6, 4, 5, 4
    q, k, v, th, w, gw, gb = rand_inputs(rng, B, H, T, d, c_q, c_k, c_h)
    st = oracle.stages(q, k, v, th, w, gw, gb, 1.0)
    np.testing.assert_allclose(st["P"].sum(-1), 1.0, rtol=0, atol=1e-13)
    want = w[0].sum(1)[:, None]          # [out head] -> constant over rows
    np.testing.assert_allclose(st["A"].sum(-1), np.broadcast_to(want, (H, T)), rtol=0, atol=1e-12)
    assert (st["P"] >= 0).all()


def test_groupnorm_statistics_and_depth_scale():
    # "Group Normalization": one group per head; with unit weight and zero
    # bias every (t, h) slice of out / depth_scale has mean 0 and variance
    # s2 / (s2 + eps) where s2 is the biased variance of the head output.
    rng = np.random.default_rng(8)
    B, H, T, d, c_q, c_k, c_h = 1, 4, 16, 12, 3, 5, 2
    q, k, v, th, w, _, _ = rand_inputs(rng, B, H, T, d, c_q, c_k, c_h)
    eps = 0.05   # large eps so that a misplaced eps is visible
    st = oracle.stages(q, k, v, th, w, np.ones(H * d), np.zeros(H * d), 0.6, gn_eps=eps)
    y = st["out"].reshape(T, H, d) / 0.6
    s2 = st["O"].var(axis=-1).T            # [T, H], biased
    np.testing.assert_allclose(y.mean(-1), 0.0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(y.var(-1), s2 / (s2 + eps), rtol=1e-11, atol=0)


def test_sigmoid_gate_scales_each_head_after_the_affine():
    # "Group Normalization with Sigmoid Gating": output = GroupNorm(concat)
    # * sigmoid(g_h) on head h, the gate taking the place of the depth scale.
    # Against the depth-scaled output with scale 1 (pinned above), head h must
    # come out multiplied by 1 / (1 + e^-g_h), computed here with numpy; a
    # nonzero bias makes a gate applied before the affine visible.
    rng = np.random.default_rng(10)
    B, H, T, d, c_q, c_k, c_h = 2, 4, 14, 8, 3, 5, 2
    q, k, v, th, w, gw, gb = rand_inputs(rng, B, H, T, d, c_q, c_k, c_h)
    gb = rng.standard_normal(H * d)
    g = np.array([-2.5, -0.3, 0.7, 3.0])
    plain = oracle.forward(q, k, v, th, w, gw, gb, 1.0).reshape(B, T, H, d)
    gated = oracle.forward(q, k, v, th, w, gw, gb, 0.0, gate=g).reshape(B, T, H, d)
    sig = 1.0 / (1.0 + np.exp(-g))
    np.testing.assert_allclose(gated, plain * sig[None, None, :, None], rtol=1e-13, atol=1e-14)
    # the sampled-row entry point agrees, and saturated gates turn heads off / fully on
    r = oracle.rows(q, k, v, th, w, gw, gb, 0.0, 1, [0, 5, 13], gate=g)
    np.testing.assert_array_equal(r, gated[1, [0, 5, 13]].reshape(3, H * d))
    off = oracle.forward(q, k, v, th, w, gw, gb, 0.0, gate=np.array([-800.0, 800.0, 0.0, 0.0]))
    off = off.reshape(B, T, H, d)
    assert np.all(off[:, :, 0] == 0.0)
    np.testing.assert_array_equal(off[:, :, 1], plain[:, :, 1])


def test_head_outputs_linear_in_mixing_weights():
    # Eq. (7) is linear in w, and so is the pre-normalisation output; summed
    # over a group it equals sum_h' P^h' (sum_h w[h][h'] V^h) (the rank
    # identity of the head-mixing discussion, with no output projection).
    rng = np.random.default_rng(9)
    B, H, T, d, c_q, c_k, c_h = 1, 2, 15, 6, 3, 5, 2
    q, k, v, th, w1, gw, gb = rand_inputs(rng, B, H, T, d, c_q, c_k, c_h)
    w2 = rng.standard_normal(w1.shape)
    O1 = oracle.stages(q, k, v, th, w1, gw, gb, 1.0)["O"]
    O2 = oracle.stages(q, k, v, th, w2, gw, gb, 1.0)["O"]
    st = oracle.stages(q, k, v, th, w1 + w2, gw, gb, 1.0)
    np.testing.assert_allclose(st["O"], O1 + O2, rtol=0, atol=1e-12)
    P = st["P"]; W = (w1 + w2)[0]
    lhs = st["O"].sum(0)
    rhs = sum(P[hp] @ sum(W[h, hp] * v[0, h] for h in range(2)) for hp in range(2))
    np.testing.assert_allclose(lhs, rhs, rtol=0, atol=1e-12)


def test_head_permutation_within_group():
    # Relabelling the heads of a group (inputs, kernels, gamma/beta and both
    # indices of w) relabels the outputs.
    rng = np.random.default_rng(10)
    B, H, T, d, c_q, c_k, c_h = 1, 4, 14, 5, 3, 3, 4
    q, k, v, th, w, gw, gb = rand_inputs(rng, B, H, T, d, c_q, c_k, c_h)
    perm = np.array([2, 0, 3, 1])
    out = oracle.forward(q, k, v, th, w, gw, gb, 0.8).reshape(B, T, H, d)
    wp = w[:, perm][:, :, perm]
    gwp = gw.reshape(H, d)[perm].reshape(-1); gbp = gb.reshape(H, d)[perm].reshape(-1)
    outp = oracle.forward(q[:, perm], k[:, perm], v[:, perm], th[perm], wp, gwp, gbp,
                          0.8).reshape(B, T, H, d)
    np.testing.assert_allclose(outp, out[:, :, perm], rtol=0, atol=1e-12)


def test_rows_and_forward_agree():
    rng = np.random.default_rng(11)
    B, H, T, d, c_q, c_k, c_h = 2, 4, 40, 8, 6, 11, 2
    q, k, v, th, w, gw, gb = rand_inputs(rng, B, H, T, d, c_q, c_k, c_h)
    out = oracle.forward(q, k, v, th, w, gw, gb, 0.8)
    idx = [0, 1, 5, 6, 20, 39]
    for b in range(B):
        r = oracle.rows(q, k, v, th, w, gw, gb, 0.8, b, idx)
        np.testing.assert_allclose(r, out[b, idx], rtol=0, atol=1e-13)


def test_workload_flop_count_uses_pages_mac_count():
    # Section 6 of the page: a 6 x 11 kernel costs 66 multiply-adds per logit.
    from convolved_logit_attention_b200.workloads import WORKLOADS
    w = WORKLOADS["longctx_4k"]
    per_logit = w.algorithmic_flops() // (w.B * w.H * w.live_logits())
    assert per_logit == 4 * w.d + 2 * 66 + 2 * w.c_h


@pytest.mark.parametrize("chunk", [1, 5, 7, 16])
def test_row_chunks_change_no_bit(chunk):
    """The full forward split into row chunks (each warming its rings up on
    the rows before it) gives the same bits as the unsplit loop, for the
    default module and for a composition with a post-softmax conv, whose
    second ring needs the longest warm-up."""
    rng = np.random.default_rng(31)
    B, H, T, d, c_q, c_k, c_h = 1, 4, 37, 8, 6, 11, 2
    q, k, v, th, w, gw, gb = rand_inputs(rng, B, H, T, d, c_q, c_k, c_h)
    th2 = 0.3 * rng.standard_normal(th.shape)
    w2 = rng.standard_normal(w.shape)
    try:
        oracle.set_row_chunk(T)
        ref = oracle.forward(q, k, v, th, w, gw, gb, 0.8)
        ref_c = oracle.forward_composed(q, k, v, th, w, th2, w2, gw, gb, 0.8)
        oracle.set_row_chunk(chunk)
        got = oracle.forward(q, k, v, th, w, gw, gb, 0.8)
        got_c = oracle.forward_composed(q, k, v, th, w, th2, w2, gw, gb, 0.8)
    finally:
        oracle.set_row_chunk(0)
    assert np.array_equal(got, ref)
    assert np.array_equal(got_c, ref_c)
