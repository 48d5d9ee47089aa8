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
