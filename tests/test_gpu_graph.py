"""The whole layer call is capturable in a CUDA graph (no synchronisation or
allocation inside), and a replay gives the same bits as the eager call, on
each FFN path: E2M1-term kernels, hybrid, and large-token kernels (with the tcgen05
router and the multi-block grouping)."""
import pytest
import torch

import datagen
from helpers import GpuLayer

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("H,E,k,I,T", [(512, 24, 4, 128, 64), (256, 12, 2, 128, 800), (256, 8, 4, 128, 4096)])
def test_layer_graph_replay_matches_eager(mx, H, E, k, I, T):
    cfg = datagen.LayerConfig("graph", H, E, k, I, T)
    layer = GpuLayer(mx, cfg, seed=4)
    x = datagen.make_x(cfg, 4, DEV)
    bias = torch.linspace(-0.3, 0.3, E, dtype=torch.float32, device=DEV)
    y_eager = torch.empty((T, H), dtype=torch.float32, device=DEV)
    y_graph = torch.full((T, H), float("nan"), dtype=torch.float32, device=DEV)
    ws = torch.empty(mx.mxmoe_workspace_size(T, H, I, E, k), dtype=torch.uint8, device=DEV)
    mx.mxmoe_layer_forward(x, layer.wg, bias, layer.ew.prepacked, I, k, y_eager, ws)  # also the first-call set-up
    torch.cuda.synchronize()
    assert mx.mxmoe_read_status(ws) == mx.OK
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            mx.mxmoe_layer_forward(x, layer.wg, bias, layer.ew.prepacked, I, k, y_graph, ws)
    g.replay()
    torch.cuda.synchronize()
    assert mx.mxmoe_read_status(ws) == mx.OK
    assert torch.equal(y_graph, y_eager)
    # new inputs in the same buffer: the replay follows them
    x.copy_(datagen.make_x(cfg, 5, DEV))
    g.replay()
    mx.mxmoe_layer_forward(x, layer.wg, bias, layer.ew.prepacked, I, k, y_eager, ws)
    torch.cuda.synchronize()
    assert torch.equal(y_graph, y_eager)
