"""The workspace-free expert FFN entry point (mxmoe_expert_ffn_noalloc).

Some callers cannot allocate device memory (their memory is owned by another
allocator's pool, or cudaMalloc's possible device synchronisation is not
allowed where they run). This variant keeps its scratch in a fixed static
device array inside the library. The test calls it through the C ABI twice in
a row, on two different inputs, and checks each result against the
workspace-based mxmoe_expert_ffn on the same input, within the tolerance the
other tests use. Named to run last, so a failure here never hides another
test's result.
"""
import numpy as np
import pytest
import torch

import datagen
import oracle
from tests.helpers import GpuLayer, TOL_RMS, max_err_over_rms

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_ffn_twice(mx):
    dev = "cuda"
    H, I, E, k, T = 512, 256, 12, 4, 24
    cfg = datagen.LayerConfig("noalloc", H, E, k, I, T)
    layer = GpuLayer(mx, cfg, seed=5)
    ws = torch.empty(mx.mxmoe_ffn_workspace_size(T, k, E, H, I), dtype=torch.uint8, device=dev)
    status = torch.full((1,), -1, dtype=torch.int32, device=dev)
    for call in range(2):
        x = datagen.make_x(cfg, 100 + call).to(dev)
        ids = datagen.make_ids(T, E, k, seed=200 + call)
        off, src, _ = oracle.permute(ids, E)  # grouping from the oracle: an input here
        off_d, src_d = torch.from_numpy(off).to(dev), torch.from_numpy(src).to(dev)
        y_ref = torch.full((T * k, H), float("nan"), dtype=torch.float32, device=dev)
        mx.mxmoe_expert_ffn(x, off_d, src_d, layer.ew.prepacked, k, E, I, y_ref, ws)
        y = torch.full((T * k, H), float("nan"), dtype=torch.float32, device=dev)
        status.fill_(-1)
        mx.mxmoe_expert_ffn_noalloc(x, off_d, src_d, layer.ew.prepacked, k, E, I, y, status)
        torch.cuda.synchronize()
        assert int(status.item()) == mx.OK
        got, ref = y.cpu().numpy(), y_ref.cpu().numpy()
        assert np.isfinite(got).all() and np.isfinite(ref).all()
        assert max_err_over_rms(got, ref.astype(np.float64)) <= TOL_RMS


def test_noalloc_rejects_sizes_beyond_its_scratch(mx):
    # 6144/2048/top-8 needs more than the fixed 8 MiB beyond 15 tokens
    assert mx.mxmoe_ffn_workspace_size(15, 8, 384, 6144, 2048) <= 8 << 20
    assert mx.mxmoe_ffn_workspace_size(16, 8, 384, 6144, 2048) > 8 << 20
    rc = mx.load().mxmoe_expert_ffn_noalloc(None, None, None, None, 16, 8, 384, 6144, 2048, None, None, None)
    assert rc == mx.ERR_WORKSPACE
    assert "8388608" in mx.last_error()
