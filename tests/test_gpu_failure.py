"""Failure detection on the GPU without a fault: every device-side wait of the
kernels is bounded, records MXMOE_ERR_TIMEOUT in a status word and returns.
Here one such wait is made to run out (its barrier never receives an arrival),
and the context must stay usable afterwards."""
import numpy as np
import pytest
import torch

import datagen
import oracle

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_bounded_wait_times_out_and_the_context_survives(mx):
    status = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    mx.mxmoe_selftest_wait_timeout(status, 20000)  # 20 ms
    end.record()
    torch.cuda.synchronize()
    assert int(status.item()) == mx.ERR_TIMEOUT
    assert start.elapsed_time(end) >= 19.0  # it waited the whole limit, not less
    # the same context still runs kernels and gets their results right
    cfg = datagen.BY_NAME["tiny"]
    l = datagen.make_logits(6, cfg.E, seed=11)
    ids = torch.empty((6, cfg.k), dtype=torch.int32, device=DEV)
    w = torch.empty((6, cfg.k), dtype=torch.float32, device=DEV)
    mx.mxmoe_route(torch.from_numpy(l).to(DEV), cfg.k, ids, w)
    ids_ref, _ = oracle.route(l, cfg.k)
    assert np.array_equal(ids.cpu().numpy(), ids_ref)
