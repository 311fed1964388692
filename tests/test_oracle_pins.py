"""Pins of the float64 CPU oracle against things other than itself.

Each test checks the oracle against what the MXFP4 format, the mathematics or
an independent library fixes: printed/hand-worked values (tests/golden), closed
forms, invariants, library routines (ml_dtypes' OCP FP4/E8M0 casts, numpy
matmul/argsort/softmax) and brute force on tiny inputs. None of them runs on a
GPU.

Pages: "MiMo-V2.5-Pro-FP4-DFlash" model card, section 2 "FP4 Quantization"
(MXFP4, block size 32); nxbn.cn MiMo-V2.5-Pro-FP4-DFlash article, architecture
section (384 experts, 8 per token, hidden 6144); alphaneural mirror, section 4
"Model Summary" (1.02T total parameters, hidden 6144, 70 layers).
"""
import math
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import datagen
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F4 = ml_dtypes.float4_e2m1fn
E8 = ml_dtypes.float8_e8m0fnu


def bf16_bits(values) -> np.ndarray:
    t = torch.tensor(np.asarray(values, np.float64), dtype=torch.float64).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_values(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def codes_of(packed: np.ndarray) -> np.ndarray:
    """Unpack nibbles: element 2j is the low nibble of byte j."""
    lo = packed & 0x0F
    hi = packed >> 4
    return np.stack([lo, hi], axis=-1).reshape(packed.shape[0], -1)


# ---------------------------------------------------------------------------
# C1: element and scale encodings
# ---------------------------------------------------------------------------
def read_e2m1_golden():
    out = {}
    with open(os.path.join(GOLDEN, "e2m1_table.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            c, v = line.split()
            out[int(c, 16)] = float(v)
    return out


def test_e2m1_table_golden():
    table = read_e2m1_golden()
    assert len(table) == 16
    for c, v in table.items():
        got = oracle.e2m1_value(c)
        assert got == v and math.copysign(1, got) == math.copysign(1, v), (c, got, v)


def test_e2m1_table_matches_ml_dtypes():
    decoded = np.arange(16, dtype=np.uint8).view(F4).astype(np.float64)
    for c in range(16):
        got = oracle.e2m1_value(c)
        assert got == decoded[c] and math.copysign(1, got) == math.copysign(1, decoded[c])


def test_e8m0_values():
    lib = np.arange(255, dtype=np.uint8).view(E8).astype(np.float64)
    for s in range(255):
        assert oracle.e8m0_value(s) == lib[s] == 2.0 ** (s - 127)
    assert math.isnan(oracle.e8m0_value(255))


def test_bf16_decode_matches_torch():
    rng = np.random.default_rng(3)
    bits = rng.integers(0, 1 << 16, size=4000, dtype=np.uint16)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]  # drop inf/nan patterns
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_to_double(int(b)) for b in bits])
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------------------
# C3: rounding rule against an independent implementation (ml_dtypes)
# ---------------------------------------------------------------------------
def test_round_ties_and_grid_against_ml_dtypes():
    grid = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    mids = [(a + b) / 2 for a, b in zip(grid, grid[1:])]
    qs = sorted(set(grid + mids + [7.0, 7.99, 8.0, 100.0, 0.1, 0.26, 0.74, 1.3, 2.6, 3.4, 4.9, 5.1]))
    rng = np.random.default_rng(5)
    qs += list(rng.uniform(0, 9, 3000))
    for q in qs:
        ref = int(np.array([q], np.float32).astype(F4).view(np.uint8)[0]) & 7
        assert oracle.e2m1_round(q) == ref, q


def test_round_equals_binade_rint():
    """E2M1 is a 1-mantissa-bit float: within each binade round(q/step)*step with
    numpy's round-half-to-even, step 0.5 below 2, 1 in [2,4), 2 above 4."""
    rng = np.random.default_rng(9)
    qs = np.concatenate([rng.uniform(0, 6, 5000), np.arange(0, 6.01, 0.125)])
    for q in qs:
        step = 0.5 if q < 2 else (1.0 if q < 4 else 2.0)
        v = min(np.rint(q / step) * step, 6.0)
        assert oracle.e2m1_value(oracle.e2m1_round(q)) == v, q


# ---------------------------------------------------------------------------
# C3: hand-worked blocks
# ---------------------------------------------------------------------------
def read_blocks():
    blocks = []
    with open(os.path.join(GOLDEN, "quant_blocks.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, s, xs, cs, dq, pk = [p.strip() for p in line.split("|")]
            blocks.append(dict(name=name, S=int(s), x=[float(v) for v in xs.split()],
                               codes=[int(c, 16) for c in cs.split()], dq=[float(v) for v in dq.split()],
                               packed=[int(b, 16) for b in pk.split()]))
    return blocks


@pytest.mark.parametrize("blk", read_blocks(), ids=lambda b: b["name"])
def test_golden_block(blk):
    x = np.zeros(32)
    n = len(blk["x"])
    x[:n] = blk["x"]
    bits = bf16_bits(x).reshape(1, 32)
    # negative zero survives the bf16 rounding
    for i, v in enumerate(blk["x"]):
        if v == 0 and math.copysign(1, v) < 0:
            bits[0, i] = 0x8000
    packed, scales = oracle.quantize(bits)
    assert scales[0, 0] == blk["S"]
    codes = codes_of(packed)[0]
    assert list(codes[:n]) == blk["codes"]
    assert not codes[n:].any()
    assert list(packed[0, : len(blk["packed"])]) == blk["packed"]
    dq = oracle.dequantize(packed, scales)[0]
    for got, want in zip(dq[:n], blk["dq"]):
        assert got == want and math.copysign(1, got) == math.copysign(1, want)


# ---------------------------------------------------------------------------
# C3: invariants
# ---------------------------------------------------------------------------
def test_exact_roundtrip_of_representable_blocks():
    rng = np.random.default_rng(11)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    rows, nblk = 64, 8
    mags = rng.integers(0, 8, size=(rows, nblk, 32))
    mags[:, :, 0] = rng.choice([6, 7], size=(rows, nblk))  # max |c| is 4 or 6
    sign = rng.integers(0, 2, size=(rows, nblk, 32))
    s = rng.integers(-60, 60, size=(rows, nblk, 1))
    v = np.where(sign == 1, -1.0, 1.0) * grid[mags] * (2.0 ** s)
    v = v.reshape(rows, nblk * 32)
    bits = bf16_bits(v)
    assert np.array_equal(bf16_values(bits), v)  # representable in bf16
    packed, scales = oracle.quantize(bits)
    dq = oracle.dequantize(packed, scales)
    assert np.array_equal(dq, v)
    assert np.array_equal(scales.astype(np.int64), (s[:, :, 0] + 127))
    want_codes = (mags | (sign << 3)).reshape(rows, -1)
    assert np.array_equal(codes_of(packed), want_codes)


def test_idempotence():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((32, 256)) * (2.0 ** rng.integers(-30, 30, size=(32, 1)))
    x[3, 0:32] = 0.0
    bits = bf16_bits(x)
    p1, s1 = oracle.quantize(bits)
    dq = oracle.dequantize(p1, s1)
    p2, s2 = oracle.quantize(bf16_bits(dq))
    assert np.array_equal(p1, p2) and np.array_equal(s1, s2)


def test_quantize_matches_ml_dtypes_cast():
    """Rounding and encoding through ml_dtypes' OCP FP4 cast, block by block."""
    rng = np.random.default_rng(13)
    x = rng.standard_normal((48, 512)) * 0.02
    x[:, 5] *= 300  # outliers
    bits = bf16_bits(x)
    xv = bf16_values(bits).reshape(48, -1, 32)
    amax = np.abs(xv).max(-1, keepdims=True)
    _, ex = np.frexp(amax)
    e = np.clip(ex - 1 - 2, -127, 127)
    q = (xv / (2.0 ** e)).astype(np.float32).astype(F4).view(np.uint8)
    packed, scales = oracle.quantize(bits)
    assert np.array_equal(scales, (e[..., 0] + 127).astype(np.uint8))
    assert np.array_equal(codes_of(packed), q.reshape(48, -1))
    # the scale byte is ml_dtypes' E8M0 encoding of 2^e
    assert np.array_equal(scales, (2.0 ** e[..., 0]).astype(np.float32).astype(E8).view(np.uint8))


# ---------------------------------------------------------------------------
# Router
# ---------------------------------------------------------------------------
def test_router_logits_vs_numpy():
    rng = np.random.default_rng(21)
    x = bf16_bits(rng.standard_normal((5, 96)))
    wg = bf16_bits(rng.standard_normal((7, 96)) * 0.02)
    bias = rng.standard_normal(7).astype(np.float32)
    got = oracle.router_logits(x, wg, bias)
    ref = bf16_values(x) @ bf16_values(wg).T + bias.astype(np.float64)
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-13)
    got0 = oracle.router_logits(x, wg, None)
    np.testing.assert_allclose(got0, bf16_values(x) @ bf16_values(wg).T, rtol=1e-13, atol=1e-13)


def test_route_all_equal():
    l = np.full((3, 384), 0.3, np.float32)
    ids, w = oracle.route(l, 8)
    assert (ids == np.arange(8)).all()
    assert (w == 0.125).all()


def test_route_vs_sort_and_softmax():
    l = datagen.make_logits(64, 384, seed=4)
    ids, w = oracle.route(l, 8)
    for t in range(l.shape[0]):
        order = np.lexsort((np.arange(384), -l[t].astype(np.float64)))[:8]
        assert list(ids[t]) == list(order), t
        p = np.exp(l[t].astype(np.float64) - l[t].max())
        p /= p.sum()
        ref = p[order] / p[order].sum()
        np.testing.assert_allclose(w[t], ref, rtol=1e-14)
        assert abs(w[t].sum() - 1.0) < 1e-14


def test_route_ties_lower_index():
    l = np.zeros((1, 16), np.float32)
    l[0, [3, 9, 12]] = 2.0
    l[0, [1, 14]] = 1.0
    ids, _ = oracle.route(l, 4)
    assert list(ids[0]) == [3, 9, 12, 1]


# ---------------------------------------------------------------------------
# C5: permute / combine
# ---------------------------------------------------------------------------
def test_permute_vs_stable_argsort():
    ids = datagen.make_ids(37, 16, 3, seed=2)
    offsets, src_row, dst_of = oracle.permute(ids, 16)
    flat = ids.ravel()
    assert np.array_equal(src_row, np.argsort(flat, kind="stable"))
    assert np.array_equal(offsets, np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=16))]))
    assert np.array_equal(dst_of[src_row], np.arange(flat.size))
    assert np.array_equal(src_row[dst_of], np.arange(flat.size))


def test_permute_empty_experts_and_single():
    ids = np.array([[5], [5], [2]], np.int32)
    offsets, src_row, dst_of = oracle.permute(ids, 8)
    assert list(offsets) == [0, 0, 0, 1, 1, 1, 3, 3, 3]
    assert list(src_row) == [2, 0, 1]
    assert list(dst_of) == [1, 2, 0]


def test_combine_identity_and_einsum():
    rng = np.random.default_rng(31)
    T, k, H = 6, 3, 10
    ids = datagen.make_ids(T, 8, k, seed=7)
    _, _, dst_of = oracle.permute(ids, 8)
    y_perm = rng.standard_normal((T * k, H))
    w = rng.random((T, k))
    y = oracle.combine(y_perm, dst_of, w, T, k)
    ref = np.einsum("tj,tjh->th", w, y_perm[dst_of].reshape(T, k, H))
    np.testing.assert_allclose(y, ref, rtol=1e-14, atol=1e-14)
    # k = 1, w = 1: the expert outputs themselves
    ids1 = np.array([[2], [0], [2]], np.int32)
    _, _, d1 = oracle.permute(ids1, 4)
    yp = rng.standard_normal((3, H))
    assert np.array_equal(oracle.combine(yp, d1, np.ones((3, 1)), 3, 1), yp[d1])


# ---------------------------------------------------------------------------
# C6: expert FFN
# ---------------------------------------------------------------------------
def test_ffn_closed_form_all_ones():
    """All codes 0x2 (1.0) and S = 127: every weight is 1, so g = u = sum(x),
    h = sum(x)^2 * sigmoid(sum(x)) and y_c = I * h."""
    H, I = 64, 32
    p13 = np.full((2 * I, H // 2), 0x22, np.uint8)
    s13 = np.full((2 * I, H // 32), 127, np.uint8)
    p2 = np.full((H, I // 2), 0x22, np.uint8)
    s2 = np.full((H, I // 32), 127, np.uint8)
    rng = np.random.default_rng(41)
    x = bf16_bits(rng.standard_normal((3, H)) * 0.1)
    y, h = oracle.expert_ffn_mxfp4(p13, s13, p2, s2, x, want_h=True)
    sx = bf16_values(x).sum(1)
    hh = sx * sx / (1 + np.exp(-sx))
    np.testing.assert_allclose(h, np.repeat(hh[:, None], I, 1), rtol=1e-12)
    np.testing.assert_allclose(y, np.repeat((I * hh)[:, None], H, 1), rtol=1e-12)


def test_ffn_gate_rows_come_first():
    """Gate rows 1.0 (code 2), up rows 2.0 (code 4): h = silu(S) * 2S; swapping
    the halves would give silu(2S) * S."""
    H, I = 32, 32
    p13 = np.concatenate([np.full((I, H // 2), 0x22, np.uint8), np.full((I, H // 2), 0x44, np.uint8)])
    s13 = np.full((2 * I, 1), 127, np.uint8)
    p2 = np.full((H, I // 2), 0x22, np.uint8)
    s2 = np.full((H, 1), 127, np.uint8)
    x = bf16_bits(np.full((1, H), 0.125))
    y, h = oracle.expert_ffn_mxfp4(p13, s13, p2, s2, x, want_h=True)
    S = 4.0
    want = S / (1 + math.exp(-S)) * 2 * S
    assert abs(h[0, 0] - want) < 1e-12
    assert abs(y[0, 0] - I * want) < 1e-9


def test_ffn_vs_numpy_bruteforce():
    rng = np.random.default_rng(43)
    H, I, n = 96, 64, 5
    w13 = bf16_bits(rng.standard_normal((2 * I, H)) * 0.05)
    w2 = bf16_bits(rng.standard_normal((H, I)) * 0.05)
    p13, s13 = oracle.quantize(w13)
    p2, s2 = oracle.quantize(w2)
    x = bf16_bits(rng.standard_normal((n, H)))
    y, h = oracle.expert_ffn_mxfp4(p13, s13, p2, s2, x, want_h=True)
    W13 = oracle.dequantize(p13, s13)
    W2 = oracle.dequantize(p2, s2)
    xv = bf16_values(x)
    g = xv @ W13[:I].T
    u = xv @ W13[I:].T
    hh = g / (1 + np.exp(-g)) * u
    np.testing.assert_allclose(h, hh, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(y, hh @ W2.T, rtol=1e-11, atol=1e-13)


# ---------------------------------------------------------------------------
# Whole layer, tiny configuration, against numpy brute force
# ---------------------------------------------------------------------------
def test_tiny_layer_vs_numpy():
    cfg = datagen.BY_NAME["tiny"]
    x = datagen.make_x(cfg, 0)
    wg = datagen.make_router_weight(cfg, 0)
    experts = []
    for e in range(cfg.E):
        p13, s13 = oracle.quantize(datagen.make_w13(cfg, e, 0))
        p2, s2 = oracle.quantize(datagen.make_w2(cfg, e, 0))
        experts.append((p13, s13, p2, s2))
    out = oracle.moe_layer(x, wg, None, lambda e: experts[e], cfg.k)
    xv = x.double().numpy()
    logits = xv @ wg.double().numpy().T
    y = np.zeros((cfg.T, cfg.H))
    for t in range(cfg.T):
        p = np.exp(logits[t] - logits[t].max())
        p /= p.sum()
        sel = np.lexsort((np.arange(cfg.E), -p))[: cfg.k]
        assert list(out["ids"][t]) == list(sel)
        w = p[sel] / p[sel].sum()
        for j, e in enumerate(sel):
            W13 = oracle.dequantize(*experts[e][:2])
            W2 = oracle.dequantize(*experts[e][2:])
            g = W13[: cfg.I] @ xv[t]
            u = W13[cfg.I:] @ xv[t]
            y[t] += w[j] * (W2 @ (g / (1 + np.exp(-g)) * u))
    np.testing.assert_allclose(out["y"], y, rtol=1e-10, atol=1e-12)


def test_layer_sizes_match_model_summary():
    """384 experts x 3 x 6144 x 2048 per layer x 70 layers ~ the 1.02T total of
    the model summary (the experts hold the vast majority of parameters)."""
    cfg = datagen.BY_NAME["verify8"]
    total = cfg.E * 3 * cfg.H * cfg.I * 70
    assert abs(total / 1.02e12 - 1) < 0.01
    assert cfg.expert_bytes == 20_054_016
