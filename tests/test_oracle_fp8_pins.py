"""Pins of the oracle's FP8 expert weights (E4M3 elements, one E8M0 scale per
32 elements along K) against things other than itself: ml_dtypes' OCP
float8_e4m3fn decode and cast, hand-worked blocks (tests/golden), exact
round trips, idempotence, closed forms and numpy brute force. CPU only.

Pages: "MiMo-V2.5-Pro-FP4-DFlash" model card, section 2 "FP4 Quantization"
(the MXFP4 experts are compared with an FP8 baseline) and introduction (8-bit
weights still cost memory bandwidth at the trillion-parameter scale). The FP8
layout is a reading (the pages give none): the MX scheme of the FP4 experts
with E4M3 elements, scale exponent floor(log2 amax) - 8.
"""
import math
import os

import ml_dtypes
import numpy as np
import pytest

import oracle
from tests.test_oracle_pins import bf16_bits, bf16_values

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F8 = ml_dtypes.float8_e4m3fn


def test_e4m3_table_matches_ml_dtypes():
    for c in range(256):
        want = float(np.array([c], np.uint8).view(F8).astype(np.float64)[0])
        got = oracle.e4m3_value(c)
        if math.isnan(want):
            assert math.isnan(got) and c in (0x7F, 0xFF)
        else:
            assert got == want and math.copysign(1, got) == math.copysign(1, want), c


def test_e4m3_closed_form():
    # normal codes: 2^(e-7) (1 + m/8); subnormals (m/8) 2^-6; largest finite 448
    assert oracle.e4m3_value(0x38) == 1.0 and oracle.e4m3_value(0x7E) == 448.0
    assert oracle.e4m3_value(0x01) == 2.0 ** -9 and oracle.e4m3_value(0x08) == 2.0 ** -6
    for e in range(1, 16):
        for m in range(8):
            if e == 15 and m == 7:
                continue
            assert oracle.e4m3_value((e << 3) | m) == 2.0 ** (e - 7) * (1 + m / 8)


def _finite_magnitudes():
    return np.array([oracle.e4m3_value(c) for c in range(0x7F)])


def test_round_every_tie_and_grid_point_against_ml_dtypes():
    mags = _finite_magnitudes()
    mids = (mags[:-1] + mags[1:]) / 2  # exact in float32: every tie
    rng = np.random.default_rng(5)
    rand = np.concatenate([rng.uniform(0, 448, 4000), rng.uniform(0, 2.0 ** -6, 1000)])
    for q in np.concatenate([mags, mids, rand]).astype(np.float32):
        want = int(np.array([q], np.float32).astype(F8).view(np.uint8)[0])
        assert oracle.e4m3_round(float(q)) == want, q


def test_round_saturates_at_448():
    for q in (448.0, 460.0, 464.0, 479.9, 511.0, 1e6):
        assert oracle.e4m3_round(q) == 0x7E


def test_round_equals_binade_rint():
    # inside binade [2^p, 2^(p+1)) (p >= -6) the grid step is 2^(p-3): nearest
    # with ties to even is numpy's rint on q / step
    rng = np.random.default_rng(6)
    for p in range(-6, 8):
        step = 2.0 ** (p - 3)
        for q in rng.uniform(2.0 ** p, 2.0 ** (p + 1), 200):
            want = np.rint(q / step) * step
            assert oracle.e4m3_value(oracle.e4m3_round(q)) == want


def read_fp8_blocks():
    blocks = []
    with open(os.path.join(GOLDEN, "quant_fp8_blocks.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, s, xs, cs, dq = [p.strip() for p in line.split("|")]
            blocks.append(dict(name=name, S=int(s), x=[float(v) for v in xs.split()],
                               codes=[int(c, 16) for c in cs.split()], dq=[float(v) for v in dq.split()]))
    return blocks


@pytest.mark.parametrize("blk", read_fp8_blocks(), ids=lambda b: b["name"])
def test_golden_fp8_block(blk):
    n = len(blk["x"])
    x = np.zeros(32)
    x[:n] = blk["x"]
    bits = bf16_bits(x).reshape(1, 32)
    assert np.array_equal(bf16_values(bits[0, :n]), np.array(blk["x"])), "golden inputs must be exact bf16 values"
    for i, v in enumerate(blk["x"]):
        if v == 0 and math.copysign(1, v) < 0:
            bits[0, i] = 0x8000
    codes, scales = oracle.quantize_fp8(bits)
    assert scales[0, 0] == blk["S"]
    assert list(codes[0, :n]) == blk["codes"]
    assert not codes[0, n:].any()
    dq = oracle.dequantize_fp8(codes, scales)[0]
    for got, want in zip(dq[:n], blk["dq"]):
        assert got == want and math.copysign(1, got) == math.copysign(1, want)


def _ml_dtypes_block_quantize(xv: np.ndarray):
    """An independent MX FP8 quantiser from ml_dtypes' E4M3 cast: per block
    e = floor(log2 amax) - 8 (numpy frexp), clamped; magnitudes clipped to 448
    (the cast itself would give NaN above 464) and cast with round to nearest
    even; the sign bit set from numpy's signbit."""
    rows, K = xv.shape
    blocks = xv.reshape(rows, K // 32, 32)
    amax = np.abs(blocks).max(axis=2)
    _, ex = np.frexp(amax)
    e = np.where(amax > 0, ex - 1 - 8, -127)
    e = np.clip(e, -127, 127)
    q = np.abs(blocks) / np.exp2(e)[..., None].astype(np.float64)
    q = np.minimum(q, 448.0)
    mag = q.astype(np.float32).astype(F8).view(np.uint8) & 0x7F
    codes = mag | np.where(np.signbit(blocks), 0x80, 0).astype(np.uint8)
    return codes.reshape(rows, K).astype(np.uint8), (e + 127).astype(np.uint8)


def test_quantize_fp8_matches_ml_dtypes():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((24, 256)) * 0.02
    x *= 2.0 ** rng.integers(-40, 40, size=(24, 1))
    x[0, :32] = 0
    x[1, 5] = -0.0
    bits = bf16_bits(x)
    bits[2, 32:64] = np.arange(1, 33)  # bf16 subnormals
    codes, scales = oracle.quantize_fp8(bits)
    want_c, want_s = _ml_dtypes_block_quantize(bf16_values(bits))
    assert np.array_equal(scales, want_s)
    assert np.array_equal(codes, want_c)


def test_exact_roundtrip_of_representable_blocks():
    # blocks c_i * 2^s with c_i on the E4M3 grid and the largest |c_i| in
    # [256, 448]: the quantiser picks e = s and reproduces every value exactly
    rng = np.random.default_rng(8)
    mags = _finite_magnitudes()
    top = mags[(mags >= 256) & (mags <= 448)]
    for s in (-60, -9, 0, 7, 60):
        c = rng.choice(mags, (16, 32)) * rng.choice([-1.0, 1.0], (16, 32))
        c[:, rng.integers(0, 32)] = rng.choice(top, 16)
        v = c * 2.0 ** s
        bits = bf16_bits(v)
        assert np.array_equal(bf16_values(bits), v)  # E4M3 x 2^s values are exact bf16 values
        codes, scales = oracle.quantize_fp8(bits)
        assert (scales == s + 127).all()
        assert np.array_equal(oracle.dequantize_fp8(codes, scales), v)


def test_idempotence():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((8, 128)) * 2.0 ** rng.integers(-30, 30, size=(8, 1))
    c1, s1 = oracle.quantize_fp8(bf16_bits(x))
    c2, s2 = oracle.quantize_fp8(bf16_bits(oracle.dequantize_fp8(c1, s1)))
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)


def test_fp8_ffn_closed_form_gate_rows_first():
    """Gate rows 1.0 (code 0x38), up rows 2.0 (0x40), S = 127, down rows 1.0:
    h = silu(S_x) * 2 S_x and y_c = I * h; swapping the halves would give
    silu(2 S_x) * S_x."""
    H, I = 64, 32
    c13 = np.concatenate([np.full((I, H), 0x38, np.uint8), np.full((I, H), 0x40, np.uint8)])
    s13 = np.full((2 * I, H // 32), 127, np.uint8)
    c2 = np.full((H, I), 0x38, np.uint8)
    s2 = np.full((H, I // 32), 127, np.uint8)
    x = bf16_bits(np.full((1, H), 0.0625))
    y, h = oracle.expert_ffn_fp8(c13, s13, c2, s2, x, want_h=True)
    S = 4.0
    want = S / (1 + math.exp(-S)) * 2 * S
    assert abs(h[0, 0] - want) < 1e-12
    assert abs(y[0, 0] - I * want) < 1e-9


def test_fp8_ffn_vs_numpy_bruteforce():
    rng = np.random.default_rng(10)
    H, I, n = 96, 64, 5
    w13 = bf16_bits(rng.standard_normal((2 * I, H)) * 0.05)
    w2 = bf16_bits(rng.standard_normal((H, I)) * 0.05)
    c13, s13 = oracle.quantize_fp8(w13)
    c2, s2 = oracle.quantize_fp8(w2)
    x = bf16_bits(rng.standard_normal((n, H)))
    y, h = oracle.expert_ffn_fp8(c13, s13, c2, s2, x, want_h=True)
    # decode independently with ml_dtypes
    W13 = c13.view(F8).astype(np.float64) * np.repeat(np.exp2(s13.astype(np.float64) - 127), 32, axis=1)
    W2 = c2.view(F8).astype(np.float64) * np.repeat(np.exp2(s2.astype(np.float64) - 127), 32, axis=1)
    xv = bf16_values(x)
    g = xv @ W13[:I].T
    u = xv @ W13[I:].T
    hh = g / (1 + np.exp(-g)) * u
    np.testing.assert_allclose(h, hh, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(y, hh @ W2.T, rtol=1e-11, atol=1e-13)


def test_fp8_layer_through_moe_layer():
    # the layer driver takes FP8 experts: k = 1 with one expert equals that expert alone
    rng = np.random.default_rng(11)
    H, I, E = 64, 32, 3
    wg = bf16_bits(rng.standard_normal((E, H)) * 0.02)
    experts = {}
    for e in range(E):
        experts[e] = oracle.quantize_fp8(bf16_bits(rng.standard_normal((2 * I, H)) * 0.05)) + \
            oracle.quantize_fp8(bf16_bits(rng.standard_normal((H, I)) * 0.05))
    x = bf16_bits(rng.standard_normal((4, H)))
    out = oracle.moe_layer(x, wg, None, lambda e: experts[e], 1, fmt="fp8")
    for t in range(4):
        e = int(out["ids"][t, 0])
        want = oracle.expert_ffn_fp8(*experts[e], x[t:t + 1])
        np.testing.assert_allclose(out["y"][t], want[0], rtol=1e-13, atol=1e-300)
