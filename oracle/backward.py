"""fp64 gradients of the Multi-Token Attention forward (the pages' default
composition), for a future backward pass.

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
    outside the map (negative padding crops)."""
    return torch.nn.functional.pad(X, (b, -b, a, -a))


def forward(q, k, v, w_kq, w_head, gn_weight, gn_bias, depth_scale, gn_eps=1e-5):
    """out [B, T, H*d] from float64 torch tensors (the layouts of the C
    oracle: q, k, v [B,H,T,d]; w_kq [H,c_q,c_k]; w_head [H/c_h,c_h,c_h];
    gn_weight, gn_bias [H*d])."""
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
    return depth_scale * y.permute(0, 2, 1, 3).reshape(B, T, H * d)


def gradients(inputs, dout, depth_scale, gn_eps=1e-5):
    """The gradient of sum(out * dout) with respect to every input: a dict
    name -> float64 array of the input's shape, for inputs a dict of arrays
    keyed by NAMES and dout [B, T, H*d]."""
    ts = {n: torch.tensor(np.asarray(inputs[n], dtype=np.float64), requires_grad=True)
          for n in NAMES}
    out = forward(*(ts[n] for n in NAMES), depth_scale, gn_eps)
    grads = torch.autograd.grad(out, [ts[n] for n in NAMES],
                                grad_outputs=torch.as_tensor(np.asarray(dout, np.float64)))
    return {n: g.numpy() for n, g in zip(NAMES, grads)}


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
