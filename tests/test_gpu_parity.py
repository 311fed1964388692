"""GPU-vs-oracle parity of every step of the MXFP4 MoE layer, through the C ABI.

Bars: quantiser bytes and scales, top-k ids and the grouping arrays are
bit-exact; floating-point outputs are within max|gpu - oracle| <= 5e-3 *
RMS(oracle) (layer and expert outputs); router logits within 1e-5 * sum|x w|
per element. Inputs come from datagen; expected values from the oracle only.
"""
import numpy as np
import pytest
import torch

import datagen
import oracle
from tests.helpers import GpuLayer, OracleExperts, THREADS, TOL_RMS, bf16_bits, max_err_over_rms

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _bf16(values):
    return torch.tensor(np.asarray(values, np.float64), dtype=torch.float64).to(torch.bfloat16)


# ---------------------------------------------------------------------------
# Quantiser
# ---------------------------------------------------------------------------
def test_quantize_golden_blocks(mx):
    from tests.test_oracle_pins import read_blocks

    blocks = read_blocks()
    x = np.zeros((len(blocks), 32))
    for i, b in enumerate(blocks):
        x[i, : len(b["x"])] = b["x"]
    w = _bf16(x)
    for i, b in enumerate(blocks):
        for j, v in enumerate(b["x"]):
            if v == 0 and np.signbit(v):
                w.view(torch.int16)[i, j] = -32768  # 0x8000
    packed, scales = mx.quantize(w.to(DEV))
    packed, scales = packed.cpu().numpy(), scales.cpu().numpy()
    for i, b in enumerate(blocks):
        assert scales[i, 0] == b["S"], b["name"]
        assert list(packed[i, : len(b["packed"])]) == b["packed"], b["name"]


def _edge_bf16(rows, K, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, K)) * 0.02
    x *= 2.0 ** rng.integers(-20, 20, size=(rows, 1))
    bits = torch.from_numpy(x).to(torch.bfloat16)
    b = bits.view(torch.int16)
    b[0, :32] = 0                         # all-zero block
    b[0, 32:64] = -32768                  # all negative-zero block
    b[1, :32] = torch.arange(1, 33)       # subnormal bf16 values
    b[1, 32:40] = torch.tensor([0x7F7F, -0x81, 0x7F00, 0x0080, -0x7F80 + 0, 0x3F80, 0x4000, 0x40C0],
                               dtype=torch.int16)  # max, -max, large, min normal, ...
    grid = torch.tensor([0, 0.5, 1, 1.5, 2, 3, 4, 6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, 7.5])
    b[2, :32] = torch.cat([grid, -grid]).to(torch.bfloat16).view(torch.int16)  # every tie
    return bits


@pytest.mark.parametrize("rows,K", [(4, 64), (37, 96), (64, 6144), (129, 2048)])
def test_quantize_bitexact(mx, rows, K):
    w = _edge_bf16(rows, K, rows + K)
    p_ref, s_ref = oracle.quantize(bf16_bits(w))
    packed, scales = mx.quantize(w.to(DEV))
    assert np.array_equal(scales.cpu().numpy(), s_ref)
    assert np.array_equal(packed.cpu().numpy(), p_ref)


def test_dequantize_exact(mx):
    w = _edge_bf16(16, 256, 5)
    p_ref, s_ref = oracle.quantize(bf16_bits(w))
    ref = oracle.dequantize(p_ref, s_ref)
    out = mx.dequantize(torch.from_numpy(p_ref).to(DEV), torch.from_numpy(s_ref).to(DEV)).cpu().numpy()
    assert np.array_equal(out.astype(np.float64), ref.astype(np.float32).astype(np.float64))


# ---------------------------------------------------------------------------
# Router
# ---------------------------------------------------------------------------
# From 512 tokens (H a multiple of 64) the router runs on tcgen05: ragged expert
# and token tiles, one K step, and the full hidden size.
@pytest.mark.parametrize("T,H,E", [(1, 64, 16), (8, 6144, 384), (37, 256, 20), (300, 512, 64), (700, 384, 200),
                                   (513, 64, 8), (1024, 6144, 384)])
def test_router_gemm(mx, T, H, E):
    cfg = datagen.LayerConfig("t", H, E, 2, 64, T)
    x = datagen.make_x(cfg, 3)
    wg = datagen.make_router_weight(cfg, 3)
    bias = torch.linspace(-1, 1, E, dtype=torch.float32)
    ref = oracle.router_logits(bf16_bits(x), bf16_bits(wg), bias.numpy())
    scale = np.abs(x.double().numpy()) @ np.abs(wg.double().numpy()).T
    logits = torch.empty((T, E), dtype=torch.float32, device=DEV)
    mx.mxmoe_router_gemm(x.to(DEV), wg.to(DEV), bias.to(DEV), logits)
    got = logits.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= 1e-5 * scale + 1e-6)


# every expert-count bin of the warp-per-token kernel (128/256/384/512/1024),
# the block kernel (E > 1024), logits rounded to few levels (many ties, which
# go to the lower expert index), and logits <= 0 whose maximum is a mix of
# -0.0 and +0.0 (equal values: index order decides)
@pytest.mark.parametrize("T,E,k,ties", [(64, 384, 8, ""), (37, 16, 2, ""), (5, 1000, 32, ""), (1, 8, 8, ""),
                                        (200, 96, 1, ""), (33, 256, 8, ""), (9, 512, 4, ""), (17, 1024, 8, ""),
                                        (3, 3000, 8, ""), (41, 384, 8, "rounded"), (7, 2500, 6, "rounded"),
                                        (19, 384, 8, "zeros"), (5, 2000, 8, "zeros")])
def test_route_bitexact(mx, T, E, k, ties):
    l = datagen.make_logits(T, E, seed=T + E)
    if ties:
        l = np.round(l * 2.0).astype(np.float32) / np.float32(2.0)
    if ties == "zeros":
        l = -np.abs(l)
        l[:, 3::7] = np.float32(-0.0)
        l[:, 5::7] = np.float32(0.0)
    ids_ref, w_ref = oracle.route(l, k)
    ids = torch.empty((T, k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, k), dtype=torch.float32, device=DEV)
    mx.mxmoe_route(torch.from_numpy(l).to(DEV), k, ids, w)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
    wg = w.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(wg - w_ref)) < 2e-6
    assert np.max(np.abs(wg.sum(1) - 1)) < 1e-6


@pytest.mark.parametrize("T,k,E", [(8, 8, 384), (37, 3, 16), (1024, 8, 384), (3000, 8, 384), (5, 2, 64)])
def test_permute_bitexact(mx, T, k, E):
    ids_np = datagen.make_ids(T, E, k, seed=T)
    off_ref, src_ref, dst_ref = oracle.permute(ids_np, E)
    ids = torch.from_numpy(ids_np).to(DEV)
    off = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    src = torch.empty(T * k, dtype=torch.int32, device=DEV)
    dst = torch.empty(T * k, dtype=torch.int32, device=DEV)
    mx.mxmoe_permute(ids, E, off, src, dst)
    assert np.array_equal(off.cpu().numpy(), off_ref)
    assert np.array_equal(src.cpu().numpy(), src_ref)
    assert np.array_equal(dst.cpu().numpy(), dst_ref)


@pytest.mark.parametrize("T,k,E,skew", [(1024, 8, 384, False), (8192, 8, 384, False), (3001, 7, 1000, False),
                                        (4097, 1, 16, False), (6000, 8, 384, True)])
def test_permute_ws_bitexact(mx, T, k, E, skew):
    # the multi-block grouping (more than 4096 pairs), ragged last block, one-pair-per-token, hot experts
    if skew:
        rng = np.random.default_rng(5)
        hot = rng.choice(E, 6, replace=False)
        ids_np = np.stack([np.concatenate([hot[:3], rng.choice(np.setdiff1d(np.arange(E), hot[:3]), k - 3, False)])
                           for _ in range(T)]).astype(np.int32)
    else:
        ids_np = datagen.make_ids(T, E, k, seed=T + 3)
    off_ref, src_ref, dst_ref = oracle.permute(ids_np, E)
    scratch = torch.empty(mx.mxmoe_permute_scratch_size(T, k, E), dtype=torch.uint8, device=DEV)
    off = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    src = torch.empty(T * k, dtype=torch.int32, device=DEV)
    dst = torch.empty(T * k, dtype=torch.int32, device=DEV)
    mx.mxmoe_permute_ws(torch.from_numpy(ids_np).to(DEV), E, off, src, dst, scratch)
    assert np.array_equal(off.cpu().numpy(), off_ref)
    assert np.array_equal(src.cpu().numpy(), src_ref)
    assert np.array_equal(dst.cpu().numpy(), dst_ref)


def test_permute_skewed(mx):
    T, k, E = 1500, 8, 384
    rng = np.random.default_rng(1)
    hot = rng.choice(E, 12, replace=False)
    ids_np = np.stack([np.concatenate([hot[:4], rng.choice(np.setdiff1d(np.arange(E), hot[:4]), k - 4, False)])
                       for _ in range(T)]).astype(np.int32)
    off_ref, src_ref, dst_ref = oracle.permute(ids_np, E)
    off = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    src = torch.empty(T * k, dtype=torch.int32, device=DEV)
    dst = torch.empty(T * k, dtype=torch.int32, device=DEV)
    mx.mxmoe_permute(torch.from_numpy(ids_np).to(DEV), E, off, src, dst)
    assert np.array_equal(off.cpu().numpy(), off_ref)
    assert np.array_equal(src.cpu().numpy(), src_ref)
    assert np.array_equal(dst.cpu().numpy(), dst_ref)


# ---------------------------------------------------------------------------
# Expert FFN (grouped), element by element against the oracle
# ---------------------------------------------------------------------------
FFN_CASES = [
    # H, I, E, k, T : several 256-row tiles along I and H, several K chunks,
    # more work items than SMs, the large-token (fp8-kind tensor-core) path from 16384 rows,
    # ragged token passes (8-token passes for T <= 8, 16-token passes
    # otherwise); H or I = 128 mod 256 gives a trailing half K chunk and, for
    # H, a down tile of 128 real rows
    (256, 128, 16, 2, 4),
    (384, 256, 6, 2, 37),     # n_e up to ~20: two 16-token passes
    (512, 512, 8, 2, 9),
    (256, 384, 3, 1, 80),     # n_e up to ~40: several passes, 3 tiles along I
    (640, 384, 5, 3, 150),
    (1024, 128, 2, 2, 1),     # one token: 7 of the 8 pass rows unused
    (1024, 1024, 64, 4, 64),  # more items than SMs in both stages
    (1024, 512, 64, 8, 8),    # ~180 items of one pass each
    (256, 128, 12, 2, 800),   # ~133 rows per expert: hybrid, experts above 128 rows on the large-token kernel
    (640, 384, 10, 2, 640),   # hybrid with ragged H and I: ~128 rows per expert, either side of the cut
    (256, 128, 7, 2, 8192),   # 16384 grouped rows: both stages on the large-token kernel, ragged passes
    (640, 384, 5, 2, 8192),   # large-token path with 3 gate/up boxes, a half-real down box and half K chunks
]


@pytest.mark.parametrize("H,I,E,k,T", FFN_CASES)
def test_expert_ffn(mx, H, I, E, k, T):
    cfg = datagen.LayerConfig("ffn", H, E, k, I, T)
    layer = GpuLayer(mx, cfg, seed=7)
    ox = OracleExperts(cfg, seed=7)
    x = datagen.make_x(cfg, 7)
    ids_np = datagen.make_ids(T, E, k, seed=T + 1)
    off, src, dst = oracle.permute(ids_np, E)
    y_ref = np.zeros((T * k, H))
    xb = bf16_bits(x)
    for e in range(E):
        rows = src[off[e]:off[e + 1]]
        if len(rows):
            y_ref[off[e]:off[e + 1]] = oracle.expert_ffn_mxfp4(*ox(e), np.ascontiguousarray(xb[rows // k]))
    ws = torch.empty(mx.mxmoe_ffn_workspace_size(T, k, E, H, I), dtype=torch.uint8, device=DEV)
    y = torch.full((T * k, H), float("nan"), dtype=torch.float32, device=DEV)
    mx.mxmoe_expert_ffn(x.to(DEV), torch.from_numpy(off).to(DEV), torch.from_numpy(src).to(DEV),
                        layer.ew.prepacked, k, E, I, y, ws)
    assert mx.mxmoe_read_status(ws) == mx.OK
    got = y.cpu().numpy()
    assert np.isfinite(got).all()
    assert max_err_over_rms(got, y_ref) <= TOL_RMS


def test_combine(mx):
    T, k, H = 33, 4, 256
    rng = np.random.default_rng(3)
    ids_np = datagen.make_ids(T, 16, k, seed=3)
    _, _, dst = oracle.permute(ids_np, 16)
    y_perm = rng.standard_normal((T * k, H)).astype(np.float32)
    w = rng.random((T, k)).astype(np.float32)
    ref = oracle.combine(y_perm.astype(np.float64), dst, w.astype(np.float64), T, k)
    y = torch.empty((T, H), dtype=torch.float32, device=DEV)
    mx.mxmoe_combine(torch.from_numpy(y_perm).to(DEV), torch.from_numpy(dst).to(DEV), torch.from_numpy(w).to(DEV), y)
    assert np.max(np.abs(y.cpu().numpy() - ref)) <= 1e-5 * np.max(np.abs(ref))


# ---------------------------------------------------------------------------
# Whole layer
# ---------------------------------------------------------------------------
def run_layer(mx, layer, x, bias, forward=None):
    cfg = layer.cfg
    T = x.shape[0]
    ws = torch.empty(mx.mxmoe_workspace_size(T, cfg.H, cfg.I, cfg.E, cfg.k), dtype=torch.uint8, device=DEV)
    y = torch.empty((T, cfg.H), dtype=torch.float32, device=DEV)
    ids = torch.empty((T, cfg.k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, cfg.k), dtype=torch.float32, device=DEV)
    (forward or mx.mxmoe_layer_forward)(x, layer.wg, bias, layer.ew.prepacked, cfg.I, cfg.k, y, ws, ids, w)
    assert mx.mxmoe_read_status(ws) == mx.OK
    return y.cpu().numpy(), ids.cpu().numpy(), w.cpu().numpy()


def check_layer(mx, layer, ox, x, bias, sample, check_bytes=False, forward=None):
    cfg = layer.cfg
    y, ids, w = run_layer(mx, layer, x.to(DEV), None if bias is None else torch.from_numpy(bias).to(DEV), forward)
    xs = x[torch.from_numpy(sample)]
    fetch = ox
    if check_bytes:
        def fetch(e):
            out = ox(e)
            gp = (layer.ew.packed13[e], layer.ew.sc13[e], layer.ew.packed2[e], layer.ew.sc2[e])
            for a, b in zip(out, gp):
                assert np.array_equal(a, b.cpu().numpy()), "quantiser bytes differ for expert %d" % e
            return out
    ref = oracle.moe_layer(xs, bf16_bits(layer.wg), bias, fetch, cfg.k, threads=THREADS)
    # near ties at the k-th logit: the GPU routes from float32 logits
    srt = -np.sort(-ref["logits"], axis=1)
    gap = srt[:, cfg.k - 1] - srt[:, cfg.k] if cfg.E > cfg.k else np.full(len(sample), np.inf)
    flagged = gap < 1e-3
    same = np.array([set(ids[t]) == set(ref["ids"][i]) for i, t in enumerate(sample)])
    assert np.all(same | flagged), "routing differs on an unflagged token"
    keep = same
    assert np.array_equal(ids[sample][keep], ref["ids"][keep])
    assert np.max(np.abs(w[sample][keep] - ref["w"][keep])) < 1e-4
    err = max_err_over_rms(y[sample][keep], ref["y"][keep])
    assert err <= TOL_RMS, err
    return dict(err=err, excluded=int((~keep).sum()), touched=ref["touched"])


def test_layer_tiny(mx):
    cfg = datagen.BY_NAME["tiny"]
    layer = GpuLayer(mx, cfg, 0)
    x = datagen.make_x(cfg, 0)
    info = check_layer(mx, layer, OracleExperts(cfg, 0), x, None, np.arange(cfg.T), check_bytes=True)
    assert info["excluded"] == 0


@pytest.mark.parametrize("T", [1, 3, 64, 200])
def test_layer_small_ragged(mx, T):
    cfg = datagen.LayerConfig("small", 512, 24, 4, 128, T)
    layer = GpuLayer(mx, cfg, 1)
    x = datagen.make_x(cfg, 1)
    bias = (np.linspace(-0.5, 0.5, cfg.E)).astype(np.float32)
    check_layer(mx, layer, OracleExperts(cfg, 1), x, bias, np.arange(T))


def test_layer_router_splits(mx):
    # 600 tokens at H 2048: the tcgen05 router in 4 K splits, summed with the bias by the routing kernel
    cfg = datagen.LayerConfig("small", 2048, 24, 4, 128, 600)
    layer = GpuLayer(mx, cfg, 2)
    x = datagen.make_x(cfg, 2)
    bias = (np.linspace(-0.5, 0.5, cfg.E)).astype(np.float32)
    check_layer(mx, layer, OracleExperts(cfg, 2), x, bias, np.arange(0, 600, 3))


def test_layer_zero_tokens(mx):
    cfg = datagen.BY_NAME["tiny"]
    layer = GpuLayer(mx, cfg, 0)
    x = torch.empty((0, cfg.H), dtype=torch.bfloat16, device=DEV)
    y = torch.empty((0, cfg.H), dtype=torch.float32, device=DEV)
    ws = torch.empty(mx.mxmoe_workspace_size(0, cfg.H, cfg.I, cfg.E, cfg.k), dtype=torch.uint8, device=DEV)
    mx.mxmoe_layer_forward(x, layer.wg, None, layer.ew.prepacked, cfg.I, cfg.k, y, ws)
    small = torch.empty(16, dtype=torch.uint8, device=DEV)
    with pytest.raises(mx.MxmoeError):
        mx.mxmoe_layer_forward(x, layer.wg, None, layer.ew.prepacked, cfg.I, cfg.k, y, small)


@pytest.fixture(scope="module")
def full_layer(mx):
    layer = GpuLayer(mx, datagen.BY_NAME["verify8"], 0)
    yield layer
    del layer
    torch.cuda.empty_cache()


@pytest.mark.slow
@pytest.mark.parametrize("name", ["verify8", "verify256", "zipf1024", "prefill8192"])
def test_layer_full_size(mx, full_layer, name):
    cfg = datagen.BY_NAME[name]
    full_layer.cfg = cfg  # same layer weights (H, E, I, seed); T differs
    x = datagen.make_x(cfg, 0)
    bias = datagen.make_router_bias(cfg, 0)
    sample = datagen.sample_tokens(cfg.T, 256, 0)
    info = check_layer(mx, full_layer, OracleExperts(cfg, 0), x, bias, sample, check_bytes=(name == "verify8"))
    print(name, info)
