"""The persistent layer kernel (mxmoe_layer_forward_persistent) against the
oracle, and against the chained launches, through the C ABI.

Below 128 tokens both paths run the same steps with the same arithmetic (the
router's tiles and split sums, the routing keys, the grouping, the E2M1-term
FFN items and the combine's slot order), so their ids, weights and outputs
must be bit-identical; at any size the outputs must meet the layer's bar
against the oracle (5e-3 * RMS, ids bit-exact away from near ties).

Page: "Xiaomi MiMo-V2.5-Pro-UltraSpeed 發佈說明" (agentlenshq.com), section
"TileRT 執行模型": a persistent engine kernel removes the gaps at operator
boundaries.
"""
import numpy as np
import pytest
import torch

import datagen
from tests.helpers import GpuLayer, OracleExperts
from tests.test_gpu_parity import check_layer

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(mx, fn, layer, x, bias):
    cfg = layer.cfg
    T = x.shape[0]
    ws = torch.empty(mx.mxmoe_workspace_size(T, cfg.H, cfg.I, cfg.E, cfg.k), dtype=torch.uint8, device=DEV)
    y = torch.full((T, cfg.H), float("nan"), dtype=torch.float32, device=DEV)
    ids = torch.empty((T, cfg.k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, cfg.k), dtype=torch.float32, device=DEV)
    fn(x, layer.wg, bias, layer.ew.prepacked, cfg.I, cfg.k, y, ws, ids, w)
    assert mx.mxmoe_read_status(ws) == mx.OK
    return y.cpu().numpy(), ids.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("H,E,k,I,T,biased", [(256, 16, 2, 128, 4, False), (512, 24, 4, 128, 1, True),
                                              (512, 24, 4, 128, 3, False), (640, 40, 8, 384, 16, True),
                                              (512, 64, 8, 256, 64, True), (1024, 384, 8, 256, 9, False)])
def test_persistent_equals_chained_bitwise(mx, H, E, k, I, T, biased):
    cfg = datagen.LayerConfig("pl", H, E, k, I, T)
    layer = GpuLayer(mx, cfg, 3)
    x = datagen.make_x(cfg, 3).to(DEV)
    bias = torch.linspace(-0.5, 0.5, E, dtype=torch.float32, device=DEV) if biased else None
    yp, ip, wp = _run(mx, mx.mxmoe_layer_forward_persistent, layer, x, bias)
    yc, ic, wc = _run(mx, mx.mxmoe_layer_forward_chained, layer, x, bias)
    assert np.array_equal(ip, ic) and np.array_equal(wp, wc)
    assert np.array_equal(yp, yc)
    # whichever path mxmoe_layer_forward takes: the same bits
    ya, _, _ = _run(mx, mx.mxmoe_layer_forward, layer, x, bias)
    assert np.array_equal(ya, yp)


def test_persistent_repeated_calls(mx):
    # the grid barrier counter starts from zero on every call; calls back to back on one stream, one workspace
    cfg = datagen.LayerConfig("pl", 512, 24, 4, 128, 8)
    layer = GpuLayer(mx, cfg, 4)
    ws = torch.empty(mx.mxmoe_workspace_size(8, 512, 128, 24, 4), dtype=torch.uint8, device=DEV)
    outs = []
    for seed in (5, 6, 5):
        x = datagen.make_x(cfg, seed).to(DEV)
        y = torch.empty((8, 512), dtype=torch.float32, device=DEV)
        mx.mxmoe_layer_forward_persistent(x, layer.wg, None, layer.ew.prepacked, 128, 4, y, ws)
        outs.append(y)
    assert mx.mxmoe_read_status(ws) == mx.OK
    assert torch.equal(outs[0], outs[2]) and not torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("T", [1, 5, 130, 256])
def test_persistent_against_oracle(mx, T):
    cfg = datagen.LayerConfig("pl", 512, 48, 6, 256, T)
    layer = GpuLayer(mx, cfg, 6)
    x = datagen.make_x(cfg, 6)
    bias = (np.linspace(-0.3, 0.3, cfg.E)).astype(np.float32)
    check_layer(mx, layer, OracleExperts(cfg, 6), x, bias, np.arange(0, T, max(1, T // 64)),
                forward=mx.mxmoe_layer_forward_persistent)


def test_persistent_rejects_sizes_on_host(mx):
    cfg = datagen.LayerConfig("pl", 256, 400, 8, 128, 4)
    lib = mx.load()
    base, big = 1 << 20, 1 << 40  # never dereferenced: rejected before anything is enqueued
    for T, E in ((257, 16), (4, 400)):
        rc = lib.mxmoe_layer_forward_persistent(base, base, None, base, T, 256, 128, E, 8, base, None, None, base, big,
                                                None)
        assert rc == mx.ERR_INVALID_SHAPE


@pytest.mark.slow
@pytest.mark.parametrize("name", ["tiny", "verify8", "verify256"])
def test_persistent_full_size(mx, name):
    cfg = datagen.BY_NAME[name]
    layer = GpuLayer(mx, cfg, 0)
    x = datagen.make_x(cfg, 0)
    info = check_layer(mx, layer, OracleExperts(cfg, 0), x, None, np.arange(cfg.T),
                       forward=mx.mxmoe_layer_forward_persistent)
    print(name, info)
    del layer
    torch.cuda.empty_cache()
