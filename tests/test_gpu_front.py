"""The front of a decode-sized layer step in one cooperative launch (router
GEMM tiles, routing, grouping and the activation terms; the path
mxmoe_layer_forward takes below 128 tokens) against the chained launches,
through the C ABI.

Both paths run the same steps with the same arithmetic (the router's tiles and
split sums, the routing keys, the grouping in pair order, the activation
digit terms), so ids, weights and outputs must be bit-identical; the local
routing (up to 64 tokens, CTA 0 alone) and the grid-wide routing (65..127
tokens) are both covered. Repeated calls on one workspace check that the grid
barrier's count starts from zero each time.

Page: "Xiaomi MiMo-V2.5-Pro-UltraSpeed 發佈說明" (agentlenshq.com), section
"TileRT 執行模型": removing the gaps at operator boundaries.
"""
import numpy as np
import pytest
import torch

import datagen
from tests.helpers import GpuLayer

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(mx, fn, layer, x, bias, ws=None):
    cfg = layer.cfg
    T = x.shape[0]
    if ws is None:
        ws = torch.empty(mx.mxmoe_workspace_size(T, cfg.H, cfg.I, cfg.E, cfg.k), dtype=torch.uint8, device=DEV)
    y = torch.full((T, cfg.H), float("nan"), dtype=torch.float32, device=DEV)
    ids = torch.empty((T, cfg.k), dtype=torch.int32, device=DEV)
    w = torch.empty((T, cfg.k), dtype=torch.float32, device=DEV)
    fn(x, layer.wg, bias, layer.ew.prepacked, cfg.I, cfg.k, y, ws, ids, w)
    assert mx.mxmoe_read_status(ws) == mx.OK
    return y.cpu().numpy(), ids.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("H,E,k,I,T,biased", [(256, 16, 2, 128, 1, False), (512, 24, 4, 128, 8, True),
                                              (640, 40, 8, 384, 64, True), (512, 64, 8, 256, 65, False),
                                              (1024, 384, 8, 256, 8, True), (512, 96, 6, 256, 127, True),
                                              (384, 32, 1, 128, 100, False)])
def test_front_equals_chained_bitwise(mx, H, E, k, I, T, biased):
    cfg = datagen.LayerConfig("fr", H, E, k, I, T)
    layer = GpuLayer(mx, cfg, 8)
    x = datagen.make_x(cfg, 8).to(DEV)
    bias = torch.linspace(-0.4, 0.4, E, dtype=torch.float32, device=DEV) if biased else None
    ya, ia, wa = _run(mx, mx.mxmoe_layer_forward, layer, x, bias)
    yc, ic, wc = _run(mx, mx.mxmoe_layer_forward_chained, layer, x, bias)
    assert np.array_equal(ia, ic) and np.array_equal(wa, wc)
    assert np.isfinite(ya).all() and np.array_equal(ya, yc)


def test_front_repeated_calls_one_workspace(mx):
    cfg = datagen.LayerConfig("fr", 512, 24, 4, 128, 8)
    layer = GpuLayer(mx, cfg, 9)
    ws = torch.empty(mx.mxmoe_workspace_size(8, 512, 128, 24, 4), dtype=torch.uint8, device=DEV)
    outs = []
    for seed in (5, 6, 5, 7, 5):
        x = datagen.make_x(cfg, seed).to(DEV)
        outs.append(_run(mx, mx.mxmoe_layer_forward, layer, x, None, ws)[0])
    assert np.array_equal(outs[0], outs[2]) and np.array_equal(outs[0], outs[4])
    assert not np.array_equal(outs[0], outs[1])
