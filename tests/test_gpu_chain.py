"""Back-to-back layer calls on one stream and one workspace, with no
synchronisation between them, give the same bits as lone calls.

The kernels of a call are chained (programmatic dependent launch): each may
begin while its predecessor still runs and reads, before waiting for it, only
what older kernels wrote (offsets, pass tables, weights). A read of a buffer
from the wrong call or before it is written would change bits here. Before
each call a torch kernel rewrites x, so the first kernel of a call must not
overlap the caller's own work either. Each FFN path: E2M1-term kernels,
hybrid, and large-token kernels (with the tcgen05 router and the multi-block
grouping)."""
import pytest
import torch

import datagen
from helpers import GpuLayer

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("H,E,k,I,T", [(512, 24, 4, 128, 64), (256, 12, 2, 128, 800), (256, 8, 4, 128, 4096)])
def test_layer_back_to_back_matches_lone_calls(mx, H, E, k, I, T):
    cfg = datagen.LayerConfig("chain", H, E, k, I, T)
    layer = GpuLayer(mx, cfg, seed=7)
    bias = torch.linspace(-0.2, 0.2, E, dtype=torch.float32, device=DEV)
    ws = torch.empty(mx.mxmoe_workspace_size(T, H, I, E, k), dtype=torch.uint8, device=DEV)
    xs = [datagen.make_x(cfg, s, DEV) for s in (11, 12, 13)]
    lone = []
    for x in xs:
        y = torch.empty((T, H), dtype=torch.float32, device=DEV)
        mx.mxmoe_layer_forward(x, layer.wg, bias, layer.ew.prepacked, I, k, y, ws)
        torch.cuda.synchronize()
        assert mx.mxmoe_read_status(ws) == mx.OK
        lone.append(y)
    xbuf = torch.empty_like(xs[0])
    ys = [torch.full((T, H), float("nan"), dtype=torch.float32, device=DEV) for _ in xs]
    for _ in range(2):
        for x, y in zip(xs, ys):
            torch.mul(x, 1, out=xbuf)  # a kernel of the caller's, just before the call
            mx.mxmoe_layer_forward(xbuf, layer.wg, bias, layer.ew.prepacked, I, k, y, ws)
    torch.cuda.synchronize()
    assert mx.mxmoe_read_status(ws) == mx.OK
    for y, ref in zip(ys, lone):
        assert torch.equal(y, ref)
