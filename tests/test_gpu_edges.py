"""Parity of the expert FFN with the oracle at the format's numeric edges, on
both tensor-core paths (the E2M1-term kernel at small token counts, the
large-token fp8-kind kernel from 16384 grouped rows), through the C ABI.

The MXFP4 format (model card, section 2 "FP4 Quantization": E2M1 elements,
one E8M0 scale per 32 values along K) reaches its edges where a block's scale
byte is 0, 1 or 252 (the quantiser's smallest and largest scales for bf16
weights: e = floor(log2 amax) - 2 is clamped at -127 and is at most 125 for
finite bf16), and where activations span many binades inside one 32-block.
Each expert here stresses one edge; its output rows are checked against the
oracle with that expert's own RMS, so that experts whose outputs are tiny or
huge are each held to the 5e-3 * RMS bar:

* tiny_w13  gate/up weights ~ N(0, 0.02) * 2^-120 (scale bytes 0..2: element
            values down to 0.5 * 2^-127, below bf16's normal range), inputs
            x ~ N(0, 1) * 2^100 so that g, u, h and y stay in float range;
* huge_w2   down weights whose every 32-block has its maximum in
            [2^127, 2^128) (scale byte 252), gate/up weights * 2^-13 so that
            h ~ 2^-30 and y stays finite;
* wide_h    every other gate row scaled by 2^-20 (h spans ~2^-20 inside its
            32-blocks);
* plain     ordinary weights, inputs whose 32-blocks span 2^0 .. 2^-24, 32-blocks
            with maxima of 2^-110, 2^-120 and 2^-126 (bf16 subnormals inside)
            next to ordinary blocks, all-zero and all -0 blocks, and all-zero
            rows.
One token per expert slot (k = 1), so each token's x can be shaped for its
expert. Expected values come from the oracle only.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import TOL_RMS, bf16_bits

pytestmark = pytest.mark.gpu
DEV = "cuda"
KINDS = ("tiny_w13", "huge_w2", "wide_h", "plain")


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _weights(kind, H, I, rng):
    w13 = rng.standard_normal((2 * I, H)) * 0.02
    w2 = rng.standard_normal((H, I)) * 0.02
    if kind == "tiny_w13":
        w13 *= 2.0 ** -120
    elif kind == "huge_w2":
        w13 *= 2.0 ** -13
        blocks = w2.reshape(H, I // 32, 32)
        amax = np.abs(blocks).max(axis=2, keepdims=True)
        w2 = (blocks / amax * 1.5 * 2.0 ** 127).reshape(H, I)  # every block's max in [2^127, 2^128)
    elif kind == "wide_h":
        w13[0:I:2] *= 2.0 ** -20  # every other gate row: h columns ~2^-20 beside ordinary ones
    return _bf16(w13), _bf16(w2)


def _x_row(kind, H, rng, j):
    x = rng.standard_normal(H)
    if kind == "tiny_w13":
        return x * 2.0 ** 100
    if kind != "plain":
        return x
    form = j % 4
    if form == 0:  # every 32-block spans 2^0 .. 2^-24
        return x * 2.0 ** (-24.0 * (np.arange(H) % 32) / 31.0)
    if form == 1:  # tiny blocks (maxima 2^-110, 2^-120, 2^-126) and zero / -0 blocks beside ordinary ones
        blocks = x.reshape(H // 32, 32).copy()
        for b, s in zip(range(0, H // 32, 5), (-110, -120, -126, None, "neg0")):
            if s is None:
                blocks[b] = 0.0
            elif s == "neg0":
                blocks[b] = -0.0
            else:
                blocks[b] = blocks[b] / np.abs(blocks[b]).max() * 2.0 ** s
        return blocks.reshape(H)
    if form == 2:  # an all-zero row
        return np.zeros(H)
    return x


@pytest.mark.parametrize("H,I,E,T,path", [
    (256, 256, 4, 64, "terms"),       # 16 tokens per expert: one 16-token pass each, E2M1-term kernel
    (384, 128, 4, 40, "terms"),       # ragged: a trailing half K chunk, a down tile of 128 real rows
    (256, 256, 4, 16384, "large"),    # 16384 grouped rows: both stages on the large-token (fp8-kind) kernel
    (384, 128, 4, 16384, "large"),    # large-token kernel with half K chunks and a half-real down box
])
def test_expert_ffn_format_edges(mx, H, I, E, T, path):
    rng = np.random.default_rng(H * 7 + T)
    kinds = [KINDS[e % 4] for e in range(E)]
    ew = mx.ExpertWeights(E, H, I, DEV)
    refs = []
    for e in range(E):
        w13, w2 = _weights(kinds[e], H, I, rng)
        ew.quantize_expert(e, w13.to(DEV), w2.to(DEV))
        p13, s13 = oracle.quantize(bf16_bits(w13))
        p2, s2 = oracle.quantize(bf16_bits(w2))
        refs.append((p13, s13, p2, s2))
    ew.prepack()
    # the construction reaches the format's edges (scale bytes from the oracle's own quantiser)
    assert (refs[0][1] == 0).any() and (refs[0][1] == 1).any()
    assert (refs[1][3] == 252).all()
    # k = 1: token t goes to expert t % E; its x row is shaped for that expert
    ids = (np.arange(T) % E).astype(np.int32).reshape(T, 1)
    x = np.stack([_x_row(kinds[t % E], H, rng, t // E) for t in range(T)])
    xb = _bf16(x)
    off, src, _ = oracle.permute(ids, E)
    ws = torch.empty(mx.mxmoe_ffn_workspace_size(T, 1, E, H, I), dtype=torch.uint8, device=DEV)
    y = torch.full((T, H), float("nan"), dtype=torch.float32, device=DEV)
    mx.mxmoe_expert_ffn(xb.to(DEV), torch.from_numpy(off).to(DEV), torch.from_numpy(src).to(DEV), ew.prepacked, 1, E,
                        I, y, ws)
    assert mx.mxmoe_read_status(ws) == mx.OK
    got = y.cpu().numpy().astype(np.float64)
    assert np.isfinite(got).all()
    xbits = bf16_bits(xb)
    for e in range(E):
        rows = src[off[e]:off[e + 1]]
        if T > 256:  # the large-token cases: a seeded sample of each expert's rows keeps the oracle quick
            pick = np.sort(np.random.default_rng(e).choice(len(rows), 256, replace=False))
            rows = rows[pick]
            grouped = off[e] + pick
        else:
            grouped = np.arange(off[e], off[e + 1])
        ref = oracle.expert_ffn_mxfp4(*refs[e], np.ascontiguousarray(xbits[rows]))
        g = got[grouped]
        zero = ~np.any(x[rows] != 0, axis=1)
        assert np.all(g[zero] == 0), "an all-zero row must give exact zeros (%s)" % kinds[e]
        rms = float(np.sqrt(np.mean(ref ** 2)))
        assert rms > 0 and np.isfinite(rms)
        err = float(np.max(np.abs(g - ref))) / rms
        assert err <= TOL_RMS, (kinds[e], path, err)
