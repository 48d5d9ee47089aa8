"""Seeded synthetic inputs for the Multi-Token Attention forward.

This module only draws random numbers and rounds them to the I/O precision;
it holds none of the method's arithmetic.  The oracle and the CUDA path both
consume exactly the arrays returned here (the oracle widens them to float64,
the GPU path uploads them as float32 or bfloat16 without further rounding).

Workloads (shapes and value structure follow the experiments described on
"Multi-Token Attention -- Paper Graph", sections 3.4 "Practical Design
Choices", 4.1 toy task, 4.3 long-context finetuning and 5 "Evaluation
Methodology"; the datasets themselves are not used, only the shapes):

  tiny_f32        fp32, B1 H4 d32 T128, (c_q,c_k,c_h) = (6,11,2)
  toy_letters     bf16, B8 H4 d64 T256, (4,15,2): c_q = L = 4 query letters,
                  c_k = 2N-1 for blocks of N = 8 letters
  pretrain_2k     bf16, B4 H16 d128 T2048, (6,11,2)
  longctx_4k      bf16, B2 H16 d128 T4096, (6,11,2), six planted needles per
                  (batch, head)
  long16k_*       bf16, B1 H16 d128 T16384, c_h in {2,4} x (c_q,c_k) in
                  {(6,11),(8,15),(2,3)}

Recipes:
  q, k, v         iid N(0,1) unless stated.
  w_kq            N(0, 0.05^2) plus 1.0 at the centre tap theta_{0,0}
                  (stored at [h][0][c_k // 2]); the identity initialisation
                  of "Practical Design Choices" plus noise.
  w_head          identity + N(0, 0.05^2) per group.
  gn_weight/bias  1 and 0 (pretrain_2k: weight N(1, 0.02^2)).
  depth_scale     0.8.
  toy_letters     letters iid uniform over 26 symbols; per head one embedding
                  E_h ~ N(0, 1/64) of shape [26, d] shared by q and k;
                  q = E_h[letter] + N(0, 0.1^2), k = E_h[letter] + N(0, 0.1^2)
                  with independent noise; v iid N(0,1).
  longctx_4k      per (b, h) six distinct key positions p ~ U[0, T-1) each
                  paired with a query position t ~ U(p, T); the key at p is
                  replaced by q_t + N(0, 0.1^2).
  w_kq_post,      the second key-query kernel and head mix of the
  w_head_post,    compositions of "Putting Everything Together: The Full MTA
  w_head_pre,     Module", the pre-softmax head mix of the logits and the 3-D
  w_kq_3d         kernel (identity on each head's own centre tap plus
                  N(0, 0.05^2) everywhere), drawn like w_kq and w_head from
                  their own stream (seed + 7919), so that the default inputs
                  stay unchanged.
"""
from dataclasses import dataclass, replace

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    d: int
    c_q: int
    c_k: int
    c_h: int
    io: str          # "f32" or "bf16"
    seed: int
    recipe: str = "iid"          # "iid", "letters" or "needles"
    gamma_std: float = 0.0
    depth_scale: float = 0.8
    gn_eps: float = 1e-5

    @property
    def G(self) -> int:
        return self.H // self.c_h

    def live_logits(self) -> int:
        """Causal (query, key) pairs per (batch, head): T (T + 1) / 2."""
        return self.T * (self.T + 1) // 2

    def algorithmic_flops(self) -> int:
        """B H L (4 d + 2 c_q c_k + 2 c_h): causal QK^T and PV, the c_q x c_k
        conv MACs per live logit and the c_h mixing MACs per head-logit
        (1 MAC = 2 FLOP)."""
        per_logit = 4 * self.d + 2 * self.c_q * self.c_k + 2 * self.c_h
        return self.B * self.H * self.live_logits() * per_logit

    def tokens(self) -> int:
        return self.B * self.T

    def composition_flops(self, comp: dict) -> int:
        """algorithmic_flops for a composition (an entry of COMPOSITIONS):
        every key-query conv costs c_q c_k MACs per live logit (the 3-D conv
        c_h c_q c_k) and every head mix c_h."""
        n_kq = sum(bool(comp.get(n)) for n in ("w_kq", "w_kq_post"))
        n_kq += self.c_h * bool(comp.get("w_kq_3d"))
        n_mix = sum(bool(comp.get(n)) for n in ("w_head_pre", "w_head", "w_head_post"))
        per_logit = 4 * self.d + 2 * n_kq * self.c_q * self.c_k + 2 * n_mix * self.c_h
        return self.B * self.H * self.live_logits() * per_logit


WEIGHT_NAMES = ("w_kq", "w_head_pre", "w_head", "w_kq_post", "w_head_post", "w_kq_3d")

# The steps of each composition: the weights it has (the others are None)
# and whether its first key-query conv uses the exact indicator of Eq. (4).
COMPOSITIONS = {
    "default": dict(w_kq=1, w_head=1),     # key-query pre-softmax, head post-softmax
    "repeat": dict(w_kq=1, w_head=1, w_kq_post=1, w_head_post=1),
    "both_post": dict(w_kq_post=1, w_head_post=1),
    "post_kq": dict(w_kq_post=1),          # the post-softmax key-query variant alone
    "mix_then_post_kq": dict(w_head=1, w_kq_post=1),
    "pre_and_post_kq": dict(w_kq=1, w_kq_post=1),
    "plain_attention": dict(),
    "both_pre": dict(w_kq=1, w_head_pre=1),  # the separable 3-D conv of the logits
    "logit_mix": dict(w_head_pre=1),       # the pre-softmax head mix alone
    "exact": dict(w_kq=1, w_head=1, exact_mask=1),
    "exact_both_pre": dict(w_kq=1, w_head_pre=1, exact_mask=1),
    "exact_repeat": dict(w_kq=1, w_head=1, w_kq_post=1, w_head_post=1, exact_mask=1),
    "conv3d": dict(w_kq_3d=1),             # one 3-D kernel over (query, key, head)
    "conv3d_exact_mix": dict(w_kq_3d=1, w_head=1, exact_mask=1),
}


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 4, 128, 32, 6, 11, 2, "f32", 0),
    "toy_letters": Workload("toy_letters", 8, 4, 256, 64, 4, 15, 2, "bf16", 1, recipe="letters"),
    "pretrain_2k": Workload("pretrain_2k", 4, 16, 2048, 128, 6, 11, 2, "bf16", 2, gamma_std=0.02),
    "longctx_4k": Workload("longctx_4k", 2, 16, 4096, 128, 6, 11, 2, "bf16", 3, recipe="needles"),
}
for _ch in (2, 4):
    for _cq, _ck in ((6, 11), (8, 15), (2, 3)):
        _n = "long16k_ch%d_%dx%d" % (_ch, _cq, _ck)
        WORKLOADS[_n] = Workload(_n, 1, 16, 16384, 128, _cq, _ck, _ch, "bf16", 4)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returned as
    float32 holding exactly representable bfloat16 values."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = ((u + 0x7FFF + lsb) >> 16) << 16
    return (u & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def _io_round(x: np.ndarray, io: str) -> np.ndarray:
    x = np.asarray(x, dtype=np.float32)
    return round_to_bf16(x) if io == "bf16" else x


def make_inputs(w: Workload, seed: int = None) -> dict:
    """Returns q, k, v [B,H,T,d] (float32 arrays holding I/O-precision values),
    w_kq [H,c_q,c_k], w_head [G,c_h,c_h], gn_weight, gn_bias [H*d] (float32),
    depth_scale (float) and gn_eps."""
    rng = np.random.default_rng(w.seed if seed is None else seed)
    B, H, T, d = w.B, w.H, w.T, w.d
    if w.recipe == "letters":
        letters = rng.integers(0, 26, size=(B, T))
        E = rng.standard_normal((H, 26, d), dtype=np.float32) / np.float32(8.0)
        base = E[np.arange(H)[None, :, None], letters[:, None, :]]        # [B,H,T,d]
        q = base + np.float32(0.1) * rng.standard_normal((B, H, T, d), dtype=np.float32)
        k = base + np.float32(0.1) * rng.standard_normal((B, H, T, d), dtype=np.float32)
        v = rng.standard_normal((B, H, T, d), dtype=np.float32)
        q, k, v = (_io_round(a, w.io) for a in (q, k, v))
    else:
        q = _io_round(rng.standard_normal((B, H, T, d), dtype=np.float32), w.io)
        k = _io_round(rng.standard_normal((B, H, T, d), dtype=np.float32), w.io)
        v = _io_round(rng.standard_normal((B, H, T, d), dtype=np.float32), w.io)
        if w.recipe == "needles":
            for b in range(B):
                for h in range(H):
                    pos = rng.choice(T - 1, size=6, replace=False)
                    for p in pos:
                        t = int(rng.integers(p + 1, T))
                        noisy = q[b, h, t] + np.float32(0.1) * rng.standard_normal(d, dtype=np.float32)
                        k[b, h, p] = _io_round(noisy, w.io)
    w_kq = np.float32(0.05) * rng.standard_normal((H, w.c_q, w.c_k), dtype=np.float32)
    w_kq[:, 0, w.c_k // 2] += np.float32(1.0)
    w_head = np.eye(w.c_h, dtype=np.float32)[None] + \
        np.float32(0.05) * rng.standard_normal((w.G, w.c_h, w.c_h), dtype=np.float32)
    if w.gamma_std > 0:
        gn_weight = (1.0 + w.gamma_std * rng.standard_normal(H * d)).astype(np.float32)
    else:
        gn_weight = np.ones(H * d, dtype=np.float32)
    gn_bias = np.zeros(H * d, dtype=np.float32)
    return {"q": q, "k": k, "v": v, "w_kq": w_kq, "w_head": w_head.astype(np.float32),
            "gn_weight": gn_weight, "gn_bias": gn_bias,
            "depth_scale": float(w.depth_scale), "gn_eps": float(w.gn_eps)}


def post_weights(w: Workload, seed: int = None) -> dict:
    """w_kq_post [H,c_q,c_k] and w_head_post [G,c_h,c_h] (float32), drawn
    like w_kq and w_head: identity plus N(0, 0.05^2)."""
    rng = np.random.default_rng((w.seed if seed is None else seed) + 7919)
    w_kq_post = np.float32(0.05) * rng.standard_normal((w.H, w.c_q, w.c_k), dtype=np.float32)
    w_kq_post[:, 0, w.c_k // 2] += np.float32(1.0)
    w_head_post = np.eye(w.c_h, dtype=np.float32)[None] + \
        np.float32(0.05) * rng.standard_normal((w.G, w.c_h, w.c_h), dtype=np.float32)
    w_head_pre = np.eye(w.c_h, dtype=np.float32)[None] + \
        np.float32(0.05) * rng.standard_normal((w.G, w.c_h, w.c_h), dtype=np.float32)
    # the 3-D kernel: identity (theta3[h][h][0][centre] = 1) plus N(0, 0.05^2)
    w_kq_3d = np.float32(0.05) * rng.standard_normal((w.G, w.c_h, w.c_h, w.c_q, w.c_k),
                                                     dtype=np.float32)
    for hh in range(w.c_h):
        w_kq_3d[:, hh, hh, 0, w.c_k // 2] += np.float32(1.0)
    return {"w_kq_post": w_kq_post, "w_head_post": w_head_post.astype(np.float32),
            "w_head_pre": w_head_pre.astype(np.float32), "w_kq_3d": w_kq_3d}


def composed_inputs(w: Workload, composition: str, seed: int = None) -> dict:
    """make_inputs plus post_weights, with the weights a composition leaves
    out set to None, and its exact_mask flag."""
    x = make_inputs(w, seed)
    x.update(post_weights(w, seed))
    comp = COMPOSITIONS[composition]
    for name in WEIGHT_NAMES:
        if not comp.get(name):
            x[name] = None
    x["exact_mask"] = bool(comp.get("exact_mask"))
    return x


def small_variant(w: Workload, **changes) -> Workload:
    """The same recipe at other sizes (used by the parity tests)."""
    return replace(w, **changes)
