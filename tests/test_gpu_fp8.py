"""GPU-vs-oracle parity of the FP8-weight variant of the layer (E4M3 expert
weights, one E8M0 scale per 32 along K), through the C ABI.

Bars as for MXFP4: quantiser codes and scales bit-exact; the expert FFN and
the whole layer within max|gpu - oracle| <= 5e-3 * RMS(oracle). Inputs come
from datagen; expected values from the oracle only.

Pages: "MiMo-V2.5-Pro-FP4-DFlash" model card, section 2 "FP4 Quantization"
(the MXFP4 experts set against an FP8 baseline); the FP8 layout is a reading
(the MX scheme with E4M3 elements), stated in include/mxmoe.h.
"""
import numpy as np
import pytest
import torch

import datagen
import oracle
from tests.helpers import THREADS, TOL_RMS, bf16_bits, max_err_over_rms

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bf16(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _edge_fp8(rows, K, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, K)) * 0.02
    x *= 2.0 ** rng.integers(-40, 40, size=(rows, 1))
    bits = _bf16(x)
    b = bits.view(torch.int16)
    b[0, :32] = 0                     # all-zero block
    b[0, 32:64] = -32768              # all negative-zero block
    b[1, :32] = torch.arange(1, 33)   # bf16 subnormals
    b[1, 32:40] = torch.tensor([0x7F7F, -0x81, 0x7F00, 0x0080, 0x3F80, 0x4000, 0x40C0, -0x4040], dtype=torch.int16)
    # every tie of one binade: 256 fixes e = 0, then the midpoints of consecutive E4M3 magnitudes below 256
    mags = np.array([oracle.e4m3_value(c) for c in range(0x7F)])
    mids = ((mags[:-1] + mags[1:]) / 2)[-31:]
    bits[2, :32] = _bf16(np.concatenate([[256.0], mids]))
    bits[3, :32] = _bf16(np.concatenate([[-256.0], -mids]))
    return bits


@pytest.mark.parametrize("rows,K", [(4, 64), (37, 96), (64, 6144), (129, 2048)])
def test_quantize_fp8_bitexact(mx, rows, K):
    w = _edge_fp8(rows, K, rows + K)
    c_ref, s_ref = oracle.quantize_fp8(bf16_bits(w))
    codes, scales = mx.quantize_fp8(w.to(DEV))
    assert np.array_equal(scales.cpu().numpy(), s_ref)
    assert np.array_equal(codes.cpu().numpy(), c_ref)


def test_dequantize_fp8_exact(mx):
    w = _edge_fp8(16, 256, 5)
    c_ref, s_ref = oracle.quantize_fp8(bf16_bits(w))
    ref = oracle.dequantize_fp8(c_ref, s_ref)
    out = mx.dequantize_fp8(torch.from_numpy(c_ref).to(DEV), torch.from_numpy(s_ref).to(DEV)).cpu().numpy()
    assert np.array_equal(out.astype(np.float64), ref.astype(np.float32).astype(np.float64))


class Fp8Layer:
    """A layer's FP8 experts generated on the device (datagen), quantised and
    prepacked by the library; the oracle quantises the same bf16 weights."""

    def __init__(self, mx, cfg, seed=0):
        self.cfg, self.seed = cfg, seed
        self.wg = datagen.make_router_weight(cfg, seed, DEV)
        self.ew = mx.ExpertWeightsFp8(cfg.E, cfg.H, cfg.I, DEV)
        for e in range(cfg.E):
            self.ew.quantize_expert(e, datagen.make_w13(cfg, e, seed, DEV), datagen.make_w2(cfg, e, seed, DEV))
        self.ew.prepack()
        torch.cuda.synchronize()
        self.cache = {}

    def oracle_expert(self, e, check_bytes=False):
        if e not in self.cache:
            c13, s13 = oracle.quantize_fp8(bf16_bits(datagen.make_w13(self.cfg, e, self.seed, DEV)))
            c2, s2 = oracle.quantize_fp8(bf16_bits(datagen.make_w2(self.cfg, e, self.seed, DEV)))
            if check_bytes:
                for a, g in zip((c13, s13, c2, s2), (self.ew.codes13[e], self.ew.sc13[e], self.ew.codes2[e],
                                                      self.ew.sc2[e])):
                    assert np.array_equal(a, g.cpu().numpy()), "FP8 quantiser bytes differ for expert %d" % e
            self.cache[e] = (c13, s13, c2, s2)
        return self.cache[e]


FP8_FFN_CASES = [
    # H, I, E, k, T: several tiles and K chunks, ragged passes, a trailing 128-row down tile (H = 128 mod 256),
    # one token, more items than SMs, and many rows per expert (several 16-token passes each)
    (256, 128, 16, 2, 4),
    (384, 256, 6, 2, 37),
    (1024, 128, 2, 2, 1),
    (640, 384, 5, 3, 150),
    (1024, 512, 64, 8, 8),
    (256, 256, 4, 2, 600),
]


@pytest.mark.parametrize("H,I,E,k,T", FP8_FFN_CASES)
def test_expert_ffn_fp8(mx, H, I, E, k, T):
    cfg = datagen.LayerConfig("ffn8", H, E, k, I, T)
    layer = Fp8Layer(mx, cfg, seed=9)
    x = datagen.make_x(cfg, 9)
    ids_np = datagen.make_ids(T, E, k, seed=T + 2)
    off, src, _ = oracle.permute(ids_np, E)
    xb = bf16_bits(x)
    y_ref = np.zeros((T * k, H))
    for e in range(E):
        rows = src[off[e]:off[e + 1]]
        if len(rows):
            y_ref[off[e]:off[e + 1]] = oracle.expert_ffn_fp8(*layer.oracle_expert(e, check_bytes=(e < 2)),
                                                             np.ascontiguousarray(xb[rows // k]))
    ws = torch.empty(mx.mxmoe_ffn_workspace_size_fp8(T, k, E, H, I), dtype=torch.uint8, device=DEV)
    y = torch.full((T * k, H), float("nan"), dtype=torch.float32, device=DEV)
    mx.mxmoe_expert_ffn_fp8(x.to(DEV), torch.from_numpy(off).to(DEV), torch.from_numpy(src).to(DEV),
                            layer.ew.prepacked, k, E, I, y, ws)
    assert mx.mxmoe_read_status(ws) == mx.OK
    got = y.cpu().numpy()
    assert np.isfinite(got).all()
    assert max_err_over_rms(got, y_ref) <= TOL_RMS


def test_expert_ffn_fp8_scale_extremes(mx):
    # gate/up weights * 2^-120 (scale bytes 0..1) with x * 2^100; down weights with every block's maximum in
    # [2^127, 2^128) (scale byte 246, the largest the quantiser gives for bf16); one token per expert slot
    H, I, E, T = 256, 256, 2, 32
    rng = np.random.default_rng(3)
    ew = mx.ExpertWeightsFp8(E, H, I, DEV)
    refs = []
    for e in range(E):
        w13 = rng.standard_normal((2 * I, H)) * 0.02
        w2 = rng.standard_normal((H, I)) * 0.02
        if e == 0:
            w13 *= 2.0 ** -120
        else:
            w13 *= 2.0 ** -13
            blk = w2.reshape(H, I // 32, 32)
            w2 = (blk / np.abs(blk).max(axis=2, keepdims=True) * 1.5 * 2.0 ** 127).reshape(H, I)
        w13b, w2b = _bf16(w13), _bf16(w2)
        ew.quantize_expert(e, w13b.to(DEV), w2b.to(DEV))
        refs.append(oracle.quantize_fp8(bf16_bits(w13b)) + oracle.quantize_fp8(bf16_bits(w2b)))
    ew.prepack()
    assert (refs[0][1] <= 1).all() and (refs[1][3] == 246).all()
    ids = (np.arange(T) % E).astype(np.int32).reshape(T, 1)
    x = rng.standard_normal((T, H)) * np.where(ids == 0, 2.0 ** 100, 1.0)
    xb = _bf16(x)
    off, src, _ = oracle.permute(ids, E)
    ws = torch.empty(mx.mxmoe_ffn_workspace_size_fp8(T, 1, E, H, I), dtype=torch.uint8, device=DEV)
    y = torch.empty((T, H), dtype=torch.float32, device=DEV)
    mx.mxmoe_expert_ffn_fp8(xb.to(DEV), torch.from_numpy(off).to(DEV), torch.from_numpy(src).to(DEV), ew.prepacked,
                            1, E, I, y, ws)
    assert mx.mxmoe_read_status(ws) == mx.OK
    got = y.cpu().numpy().astype(np.float64)
    for e in range(E):
        rows = src[off[e]:off[e + 1]]
        ref = oracle.expert_ffn_fp8(*refs[e], np.ascontiguousarray(bf16_bits(xb)[rows]))
        assert max_err_over_rms(got[off[e]:off[e + 1]], ref) <= TOL_RMS, e


def _check_layer_fp8(mx, layer, x, bias, sample, check_bytes=False):
    cfg = layer.cfg
    T = x.shape[0]
    ws = torch.empty(mx.mxmoe_workspace_size_fp8(T, cfg.H, cfg.I, cfg.E, cfg.k), dtype=torch.uint8, device=DEV)
    y = torch.empty((T, cfg.H), dtype=torch.float32, device=DEV)
    ids = torch.empty((T, cfg.k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, cfg.k), dtype=torch.float32, device=DEV)
    mx.mxmoe_layer_forward_fp8(x.to(DEV), layer.wg, None if bias is None else torch.from_numpy(bias).to(DEV),
                               layer.ew.prepacked, cfg.I, cfg.k, y, ws, ids, w)
    assert mx.mxmoe_read_status(ws) == mx.OK
    y, ids = y.cpu().numpy(), ids.cpu().numpy()
    xs = x[torch.from_numpy(sample)]
    ref = oracle.moe_layer(xs, bf16_bits(layer.wg), bias, lambda e: layer.oracle_expert(e, check_bytes), cfg.k,
                           threads=THREADS, fmt="fp8")
    srt = -np.sort(-ref["logits"], axis=1)
    flagged = (srt[:, cfg.k - 1] - srt[:, cfg.k]) < 1e-3
    same = np.array([set(ids[t]) == set(ref["ids"][i]) for i, t in enumerate(sample)])
    assert np.all(same | flagged), "routing differs on an unflagged token"
    err = max_err_over_rms(y[sample][same], ref["y"][same])
    assert err <= TOL_RMS, err
    return err


def test_layer_fp8_tiny(mx):
    cfg = datagen.BY_NAME["tiny"]
    layer = Fp8Layer(mx, cfg, 0)
    _check_layer_fp8(mx, layer, datagen.make_x(cfg, 0), None, np.arange(cfg.T), check_bytes=True)


@pytest.mark.slow
def test_layer_fp8_verify8_full_size(mx):
    # the 6144/384/top-8/2048 layer with FP8 experts, one verify block of 8 tokens, every touched expert's
    # quantiser bytes compared
    cfg = datagen.BY_NAME["verify8"]
    layer = Fp8Layer(mx, cfg, 0)
    _check_layer_fp8(mx, layer, datagen.make_x(cfg, 0), None, np.arange(cfg.T), check_bytes=True)
    del layer
    torch.cuda.empty_cache()
