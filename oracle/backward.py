"""fp64 gradients of the Multi-Token Attention forward (the pages' default
composition, with the depth scale or the sigmoid gate), the reference of the
CUDA backward pass.

TEST INFRASTRUCTURE ONLY: like the rest of this package, only the test suite
may call it; the CUDA library never imports it.

The pages give no backward pass; their cost table is for training ("Article
Overview: Multi-Token Attention", section 6), so the gradients are those of
the forward they define, with nothing else.  `forward` restates that forward
with plain torch ops on materialised T x T maps, in float64:

  [MHA]  A^ = Q K^T / sqrt(d)                  ("Multi-Token Attention --
                                                 Paper Graph", section 3.4)
  [KQ5]  A0 = Mask_0(A^); C = Conv2d_theta(A0) with the index ranges of
         Eq. (4) and zero padding; Mask_-inf; softmax over keys
  [HM7]  A^h_new = sum_h' w[h][h'] P^h' within each group of c_h heads
         ("Head Mixing Convolution", Eq. (7), after the softmax)
  [GN]   per head GroupNorm over d (biased variance, eps inside the root),
         per-channel gamma and beta over the H*d concatenation, times the
         depth scale ("Group Normalization with Sigmoid Gating"; "Article
         Overview", section 2)

and `gradients` differentiates it with torch.autograd (a library primitive
serving as the chain rule).  The restatement is checked against the C
oracle's forward, and the gradients against central finite differences of
the C oracle, in tests/test_oracle_backward_pins.py.
"""
import math

import numpy as np
import torch

NAMES = ("q", "k", "v", "w_kq", "w_head", "gn_weight", "gn_bias")


def _shift(X, a, b):
    """Y[..., i, j] = X[..., i - a, j - b], zero where i - a or j - b falls
    outside the map (negative padding crops); a shift by the map's whole
    height or width or more leaves only zeros."""
    if abs(a) >= X.shape[-2] or abs(b) >= X.shape[-1]:
        return torch.zeros_like(X)
    return torch.nn.functional.pad(X, (b, -b, a, -a))


def _out_scale(depth_scale, gate, H):
    """The per-head output scale: the depth scale ("Article Overview",
    section 2), or sigmoid(g_h) with a gate ("Group Normalization with
    Sigmoid Gating"); shaped to broadcast over [B, H, T, d]."""
    if gate is None:
        return depth_scale
    return torch.sigmoid(gate).view(1, H, 1, 1)


def forward(q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, gn_eps=1e-5, gate=None):
    """out [B, T, H*d] from float64 torch tensors (the layouts of the C
    oracle: q, k, v [B,H,T,d]; w_kq [H,c_q,c_k]; w_head [H/c_h,c_h,c_h];
    gn_weight, gn_bias [H*d]; gate [H] or None)."""
    B, H, T, d = q.shape
    _, c_q, c_k = w_kq.shape
    c_h = w_head.shape[-1]
    G = H // c_h
    causal = torch.ones(T, T, dtype=torch.bool).tril()
    logits = q @ k.transpose(-1, -2) / math.sqrt(d)                    # [MHA]
    A0 = torch.where(causal, logits, torch.zeros((), dtype=q.dtype))   # Mask_0
    C = torch.zeros_like(A0)
    for ip in range(c_q):                                              # Eq. (4)
        for jj in range(c_k):
            jp = jj - c_k // 2
            C = C + w_kq[:, ip, jj].view(1, H, 1, 1) * _shift(A0, ip, jp)
    C = C.masked_fill(~causal, float("-inf"))                          # Mask_-inf
    P = torch.softmax(C, dim=-1)
    A = torch.einsum("goi,bgitj->bgotj", w_head, P.reshape(B, G, c_h, T, T))  # [HM7]
    O = A.reshape(B, H, T, T) @ v                                      # [B,H,T,d]
    mean = O.mean(dim=-1, keepdim=True)                                # [GN]
    var = ((O - mean) ** 2).mean(dim=-1, keepdim=True)
    xhat = (O - mean) / torch.sqrt(var + gn_eps)
    y = xhat * gn_weight.view(H, 1, d) + gn_bias.view(H, 1, d)
    y = _out_scale(depth_scale, gate, H) * y
    return y.permute(0, 2, 1, 3).reshape(B, T, H * d)


def _leaves(inputs, gate):
    ts = {n: torch.tensor(np.asarray(inputs[n], dtype=np.float64), requires_grad=True)
          for n in NAMES}
    if gate is not None:
        ts["gate"] = torch.tensor(np.asarray(gate, dtype=np.float64), requires_grad=True)
    return ts


def gradients(inputs, dout, depth_scale, gn_eps=1e-5, gate=None):
    """The gradient of sum(out * dout) with respect to every input: a dict
    name -> float64 array of the input's shape, for inputs a dict of arrays
    keyed by NAMES and dout [B, T, H*d].  With gate [H] (the sigmoid gate in
    place of the depth scale) the dict also holds "gate"."""
    ts = _leaves(inputs, gate)
    out = forward(*(ts[n] for n in NAMES), depth_scale, gn_eps, gate=ts.get("gate"))
    names = list(ts)
    grads = torch.autograd.grad(out, [ts[n] for n in names],
                                grad_outputs=torch.as_tensor(np.asarray(dout, np.float64)))
    return {n: g.numpy() for n, g in zip(names, grads)}


def forward_rows(q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, rows, gn_eps=1e-5,
                 gate=None):
    """out[:, rows, :] ([B, len(rows), H*d]) of the same forward, computed
    from only what those rows depend on: for query row i, the masked logit
    rows i - c_q + 1 .. i over the keys 0 .. i (Mask_0 zeroes every key past
    its own row, and Eq. (4)'s taps reach keys j - j' <= i + floor(c_k/2)
    only through such zeros), the Eq. (4) convolution at the keys j <= i,
    softmax, Eq. (7) mix, A V over the keys j <= i and the GroupNorm.  The
    gradient of sum(out[:, rows] * dout_rows) through it is the full
    forward's gradient for an upstream gradient that is zero off `rows`."""
    B, H, T, d = q.shape
    _, c_q, c_k = w_kq.shape
    c_h = w_head.shape[-1]
    G = H // c_h
    R = c_k // 2
    outs = []
    for i in rows:
        n = i + 1                                          # keys 0 .. i
        r_idx = [i - ip for ip in range(c_q)]              # logit rows i - i'
        A0 = []
        for r in r_idx:
            if r < 0:
                A0.append(torch.zeros(B, H, n, dtype=q.dtype))
                continue
            row = (q[:, :, r, :].unsqueeze(-2) @ k[:, :, :n, :].transpose(-1, -2)).squeeze(-2)
            row = row / math.sqrt(d)
            keep = torch.arange(n) <= r                    # Mask_0
            A0.append(torch.where(keep, row, torch.zeros((), dtype=q.dtype)))
        C = torch.zeros(B, H, n, dtype=q.dtype)
        for ip in range(c_q):
            for jj in range(c_k):
                jp = jj - R                                # C[j] += theta A0[i-ip][j-jp]
                src = A0[ip]
                if jp >= 0:
                    shifted = torch.nn.functional.pad(src, (jp, 0))[..., :n]
                else:
                    shifted = torch.nn.functional.pad(src, (0, -jp))[..., -jp:]
                C = C + w_kq[:, ip, jj].view(1, H, 1) * shifted
        P = torch.softmax(C, dim=-1)                       # keys j <= i only
        A = torch.einsum("goi,bgij->bgoj", w_head, P.reshape(B, G, c_h, n)).reshape(B, H, n)
        O = (A.unsqueeze(-2) @ v[:, :, :n, :]).squeeze(-2)  # [B, H, d]
        mean = O.mean(dim=-1, keepdim=True)
        var = ((O - mean) ** 2).mean(dim=-1, keepdim=True)
        y = (O - mean) / torch.sqrt(var + gn_eps) * gn_weight.view(H, d) + gn_bias.view(H, d)
        scale = depth_scale if gate is None else torch.sigmoid(gate).view(1, H, 1)
        outs.append((scale * y).reshape(B, H * d))
    return torch.stack(outs, dim=1)


def gradients_rows(inputs, rows, dout_rows, depth_scale, gn_eps=1e-5, gate=None):
    """gradients() for an upstream gradient that is zero except at the query
    rows `rows`, where it is dout_rows [B, len(rows), H*d]; computed through
    forward_rows, so that large T stays cheap."""
    ts = _leaves(inputs, gate)
    out = forward_rows(*(ts[n] for n in NAMES), depth_scale, rows, gn_eps, gate=ts.get("gate"))
    names = list(ts)
    grads = torch.autograd.grad(out, [ts[n] for n in names],
                                grad_outputs=torch.as_tensor(np.asarray(dout_rows, np.float64)))
    return {n: g.numpy() for n, g in zip(names, grads)}


# Every composition of "Putting Everything Together: The Full MTA Module":
# the weights are those of the C oracle's composed entry.
COMPOSED_NAMES = ("q", "k", "v", "w_kq", "w_kq_3d", "w_head_pre", "w_head", "w_kq_post",
                  "w_head_post", "gn_weight", "gn_bias")


def _conv(X, th, exact):
    """Eq. (4) taps over the map X [B,H,T,T] with th [H,c_q,c_k]; with exact,
    the tap (i', j') of output (i, j) is kept only for key j - j' <= i (the
    indicator), X then holding the unmasked logits."""
    B, H, T, _ = X.shape
    _, c_q, c_k = th.shape
    I = torch.arange(T).view(T, 1)
    J = torch.arange(T).view(1, T)
    Y = torch.zeros_like(X)
    for ip in range(c_q):
        for jj in range(c_k):
            jp = jj - c_k // 2
            S = _shift(X, ip, jp)
            if exact:
                S = torch.where(J - jp <= I, S, torch.zeros((), dtype=X.dtype))
            Y = Y + th[:, ip, jj].view(1, H, 1, 1) * S
    return Y


def _mix(X, w):
    B, H, T, _ = X.shape
    G, c_h = w.shape[0], w.shape[-1]
    return torch.einsum("goi,bgitj->bgotj", w, X.reshape(B, G, c_h, T, T)).reshape(B, H, T, T)


def forward_composed(t, depth_scale, exact_mask=False, gn_eps=1e-5):
    """out [B, T, H*d] of a composition: t maps COMPOSED_NAMES to float64
    tensors or None (a step left out), in the C oracle's order: Mask_0 (or,
    with exact_mask, the unmasked logits under Eq. (4)'s indicator),
    [w_kq or the 3-D kernel w_kq_3d], [w_head_pre on the logits], Mask_-inf,
    softmax, [w_head], [w_kq_post on the probabilities, Mask_0],
    [w_head_post], A V, GroupNorm, depth scale."""
    q, k, v = t["q"], t["k"], t["v"]
    B, H, T, d = q.shape
    causal = torch.ones(T, T, dtype=torch.bool).tril()
    zero = torch.zeros((), dtype=q.dtype)
    logits = q @ k.transpose(-1, -2) / math.sqrt(d)
    A0 = torch.where(causal, logits, zero)
    src = logits if exact_mask else A0
    if t.get("w_kq_3d") is not None:                 # sum over the group's input heads
        w3 = t["w_kq_3d"]
        G, c_h = w3.shape[:2]
        parts = []
        for g in range(G):
            for ho in range(c_h):
                acc = torch.zeros_like(A0[:, 0])
                for hi in range(c_h):
                    hs = g * c_h + hi
                    acc = acc + _conv(src[:, hs:hs + 1], w3[g, ho, hi].unsqueeze(0),
                                      exact_mask)[:, 0]
                parts.append(acc)
        C = torch.stack(parts, dim=1)
    elif t.get("w_kq") is not None:
        C = _conv(src, t["w_kq"], exact_mask)
    else:
        C = A0
    if t.get("w_head_pre") is not None:
        C = _mix(C, t["w_head_pre"])
    P = torch.softmax(C.masked_fill(~causal, float("-inf")), dim=-1)
    A = _mix(P, t["w_head"]) if t.get("w_head") is not None else P
    if t.get("w_kq_post") is not None:
        A = torch.where(causal, _conv(A, t["w_kq_post"], False), zero)
    if t.get("w_head_post") is not None:
        A = _mix(A, t["w_head_post"])
    O = A @ v
    mean = O.mean(dim=-1, keepdim=True)
    var = ((O - mean) ** 2).mean(dim=-1, keepdim=True)
    y = (O - mean) / torch.sqrt(var + gn_eps) * t["gn_weight"].view(H, 1, d) \
        + t["gn_bias"].view(H, 1, d)
    return depth_scale * y.permute(0, 2, 1, 3).reshape(B, T, H * d)


def gradients_composed(inputs, dout, depth_scale, exact_mask=False, gn_eps=1e-5):
    """Gradients of sum(out * dout) for a composition: a dict name -> array
    for every input in COMPOSED_NAMES that is not None."""
    ts = {n: (None if inputs.get(n) is None else
              torch.tensor(np.asarray(inputs[n], dtype=np.float64), requires_grad=True))
          for n in COMPOSED_NAMES}
    out = forward_composed(ts, depth_scale, exact_mask, gn_eps)
    live = [n for n in COMPOSED_NAMES if ts[n] is not None]
    grads = torch.autograd.grad(out, [ts[n] for n in live],
                                grad_outputs=torch.as_tensor(np.asarray(dout, np.float64)))
    return {n: g.numpy() for n, g in zip(live, grads)}
