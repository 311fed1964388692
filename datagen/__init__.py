"""Seeded synthetic inputs for the MXFP4 MoE expert layer.

This module only draws random numbers; it holds none of the layer's
arithmetic (no quantisation, routing, GEMM or combine). Both the CUDA library's
tests/benchmark and the CPU oracle take their inputs from here.

Workloads (sizes from the pages: 384 experts, 8 active per token and hidden
size 6144 in the nxbn.cn MiMo-V2.5-Pro-FP4-DFlash article's architecture
section; the verify block of 8 tokens from the model card's section 3 and its
``--speculative-num-draft-tokens 8`` deployment flag; the expert intermediate
size 2048 is a synthetic choice that is consistent with "1.02T" total
parameters in the model summary, 384 * 3 * 6144 * 2048 * 70 layers = 1.015T):

* ``tiny``        H 256,  E 16,  k 2, I 128,  T 4
* ``verify8``     H 6144, E 384, k 8, I 2048, T 8      (one verify block)
* ``verify256``   same layer, T 256 (32 sequences x 8-token blocks)
* ``zipf1024``    same layer, T 1024, per-expert router bias so that expert
                  popularity follows Zipf(s=1.2)
* ``prefill8192`` same layer, T 8192

Block verification (``make_verify_inputs``): B sequences, each a block of K
drafted tokens over a vocabulary of V. The full-size vocabulary 152064 is a
stand-in: the pages name the drafter's mask token id 151669 (nxbn.cn article,
DFlash configuration), so the vocabulary holds at least 151670 entries; 152064
rounds that up to a multiple of 256. B = 1 and 32 match the verify8 and
verify256 token counts (8 and 256 tokens = 1 and 32 blocks of 8).

Distributions: activations x ~ N(0, 1), router weights ~ N(0, 0.02), expert
weights ~ N(0, 0.02), each drawn in float32 by a seeded torch generator and
rounded to bf16 (round to nearest even). Each tensor (and each expert's
tensors) has its own seed, so one expert can be regenerated without the rest.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    H: int  # hidden size
    E: int  # number of experts
    k: int  # experts per token
    I: int  # expert intermediate size
    T: int  # tokens in the call
    zipf_s: float | None = None  # router-bias popularity skew, None = no bias

    @property
    def expert_bytes(self) -> int:
        """MXFP4 bytes of one expert: 3*H*I elements at 4 bits plus one scale byte per 32."""
        n = 3 * self.H * self.I
        return n // 2 + n // 32


CONFIGS = [
    LayerConfig("tiny", 256, 16, 2, 128, 4),
    LayerConfig("verify8", 6144, 384, 8, 2048, 8),
    LayerConfig("verify256", 6144, 384, 8, 2048, 256),
    LayerConfig("zipf1024", 6144, 384, 8, 2048, 1024, zipf_s=1.2),
    LayerConfig("prefill8192", 6144, 384, 8, 2048, 8192),
]
BY_NAME = {c.name: c for c in CONFIGS}

_TAGS = {"x": 1, "wg": 2, "w13": 3, "w2": 4, "bias": 5, "logits": 6, "ids": 7, "misc": 8, "verify": 9}


def _seed(seed: int, tag: str, idx: int = 0) -> int:
    return (int(seed) * 1_000_003 + _TAGS[tag] * 10_007 + int(idx) * 7 + 12345) & 0x7FFF_FFFF_FFFF_FFFF


def _normal(shape, std: float, seed: int, device) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def make_x(cfg: LayerConfig, seed: int = 0, device="cpu", T: int | None = None) -> torch.Tensor:
    return _normal((cfg.T if T is None else T, cfg.H), 1.0, _seed(seed, "x"), device)


def make_router_weight(cfg: LayerConfig, seed: int = 0, device="cpu") -> torch.Tensor:
    return _normal((cfg.E, cfg.H), 0.02, _seed(seed, "wg"), device)


def make_w13(cfg: LayerConfig, e: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """bf16 [2I, H]: rows 0..I-1 gate projection, rows I..2I-1 up projection."""
    return _normal((2 * cfg.I, cfg.H), 0.02, _seed(seed, "w13", e), device)


def make_w2(cfg: LayerConfig, e: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """bf16 [H, I]: down projection."""
    return _normal((cfg.H, cfg.I), 0.02, _seed(seed, "w2", e), device)


def make_router_bias(cfg: LayerConfig, seed: int = 0) -> np.ndarray | None:
    """float32 [E] per-expert router bias giving Zipf(s) expert popularity.

    Calibrated on surrogate logits with the same distribution as the real
    ones: for fixed x the logits x.w_e of different experts are independent
    N(0, 0.02^2 |x|^2) with |x|^2 ~ H, so surrogate logits are iid
    N(0, 0.0004 H). Ranks are a seeded permutation; targets are
    T*k*r^-s / sum, water-filled under the cap T (an expert takes a token at
    most once); then 60 damped fixed-point steps move each bias by
    0.5*(ln(target+0.5) - ln(count+0.5)).
    """
    if cfg.zipf_s is None:
        return None
    rng = np.random.default_rng(_seed(seed, "bias"))
    E, T, k = cfg.E, cfg.T, cfg.k
    ranks = rng.permutation(E) + 1.0
    p = ranks ** (-cfg.zipf_s)
    p /= p.sum()
    target = T * k * p
    for _ in range(64):  # water-fill under the per-expert cap T
        over = target > T
        if not over.any():
            break
        excess = (target[over] - T).sum()
        target[over] = T
        free = ~over & (target < T)
        target[free] += excess * target[free] / target[free].sum()
    sigma = np.sqrt(0.0004 * cfg.H)
    surrogate = rng.standard_normal((T, E)) * sigma
    b = -cfg.zipf_s * np.log(ranks) * sigma
    for _ in range(60):
        sel = np.argpartition(-(surrogate + b), k - 1, axis=1)[:, :k]
        cnt = np.bincount(sel.ravel(), minlength=E).astype(np.float64)
        b += 0.5 * (np.log(target + 0.5) - np.log(cnt + 0.5))
    return b.astype(np.float32)


def make_logits(T: int, E: int, seed: int = 0, ties: bool = True) -> np.ndarray:
    """float32 [T, E] router-logit-like values N(0, 1.6^2) for routing tests.

    With ``ties``: row 0 all equal, row 1 with a block of 12 equal maxima, and
    every third row copying a few values within itself to plant exact ties.
    """
    rng = np.random.default_rng(_seed(seed, "logits"))
    l = (rng.standard_normal((T, E)) * 1.6).astype(np.float32)
    if ties and T > 0:
        l[0, :] = np.float32(0.75)
        if T > 1:
            l[1, : min(12, E)] = np.float32(3.0)
        for t in range(2, T, 3):
            src = rng.integers(0, E, size=4)
            dst = rng.integers(0, E, size=4)
            l[t, dst] = l[t, src]
    return l


def make_ids(T: int, E: int, k: int, seed: int = 0) -> np.ndarray:
    """int32 [T, k]: k distinct random experts per token (a routing outcome)."""
    rng = np.random.default_rng(_seed(seed, "ids"))
    return np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)


def sample_tokens(T: int, n: int = 256, seed: int = 0) -> np.ndarray:
    """Seeded sorted sample of min(n, T) distinct token indices."""
    if n >= T:
        return np.arange(T)
    rng = np.random.default_rng(int(seed) + 1)
    return np.sort(rng.choice(T, n, replace=False))


VERIFY_VOCAB = 152064


def make_verify_inputs(B: int, K: int, V: int, seed: int = 0, draft_noise: float = 0.4):
    """Synthetic inputs of a block verification: float32 backbone logits
    [B, K+1, V] (N(0, 1) plus, per row, one token raised by U(5, 12) so that
    rows are peaked like a language model's), float32 drafter logits [B, K, V]
    (the backbone's first K rows plus N(0, draft_noise^2)), int32 draft tokens
    [B, K] (the argmax of each drafter row) and float32 uniforms [B, K+1] in
    [0, 1). At V = 152064 these give mean accepted lengths of about 4
    (sampling at temperature 1) and 6.4 (greedy), inside the 3.18-6.30 range
    of the acceptance-length table on the model card (section 3). Only random
    draws and an argmax; no verification arithmetic."""
    rng = np.random.default_rng(_seed(seed, "verify"))
    z = rng.standard_normal((B, K + 1, V), dtype=np.float32)
    top = rng.integers(0, V, (B, K + 1))
    boost = rng.uniform(5.0, 12.0, (B, K + 1)).astype(np.float32)
    np.put_along_axis(z, top[..., None], np.take_along_axis(z, top[..., None], 2) + boost[..., None], 2)
    w = z[:, :K] + rng.standard_normal((B, K, V), dtype=np.float32) * np.float32(draft_noise)
    d = np.argmax(w, axis=2).astype(np.int32)
    u = rng.random((B, K + 1), dtype=np.float32)
    u = np.minimum(u, np.float32(1.0) - np.float32(2.0**-24))
    return z, w.astype(np.float32), d, u
