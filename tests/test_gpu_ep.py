"""The expert-parallel layer's GPU steps against the oracle on one GPU: G
simulated ranks, each with its own tokens and its own shard of the experts
(prepacked separately), run every compute step through the C ABI
(ep.LibOps: router, route, grouping, mxmoe_ep_dispatch, mxmoe_ep_expert_ffn,
mxmoe_combine) rank after rank, while the test moves the buffers between them
the way the two all-to-all exchanges would. Each rank's output must match the
oracle's whole layer on that rank's tokens (5e-3 * RMS; ids bit-exact away
from near ties), and the dispatch's bookkeeping must match what the grouping
implies (bit-exact).

Page: the SGLang launch in the "MiMo-V2.5-Pro-FP4-DFlash" model card's
deployment section serves the model with --ep-size 16.
"""
import numpy as np
import pytest
import torch

import datagen
import oracle
from mxfp4_quantized_moe_router_b200 import ep
from tests.helpers import OracleExperts, THREADS, TOL_RMS, bf16_bits, max_err_over_rms

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _shards(mx, cfg, G, seed):
    """Each simulated rank's prepacked expert shard, quantised by the library."""
    shards = []
    for g in range(G):
        e0, e1 = ep.expert_range(cfg.E, G, g)
        ew = mx.ExpertWeights(e1 - e0, cfg.H, cfg.I, DEV)
        for j, e in enumerate(range(e0, e1)):
            ew.quantize_expert(j, datagen.make_w13(cfg, e, seed, DEV), datagen.make_w2(cfg, e, seed, DEV))
        ew.prepack()
        shards.append(ew.prepacked)
    return shards


@pytest.mark.parametrize("H,E,k,I,G,T", [(256, 16, 2, 128, 2, 6), (512, 24, 4, 256, 4, 40), (256, 32, 8, 128, 8, 3),
                                         (384, 64, 8, 256, 4, 200)])
def test_ep_layer_simulated_ranks(mx, H, E, k, I, G, T):
    cfg = datagen.LayerConfig("ep", H, E, k, I, T)
    seed = 5
    wg = datagen.make_router_weight(cfg, seed, DEV)
    shards = _shards(mx, cfg, G, seed)
    ops = ep.LibOps(H, I, E, k)
    xs = [datagen.make_x(cfg, 200 + g, T=T + 3 * g) for g in range(G)]  # ranks hold different token counts
    state = []
    for g in range(G):  # sender side of every rank
        x = xs[g].to(DEV)
        ids, w = ops.route(x, wg, None)
        offsets, src_row, dst_of = ops.group(ids)
        send_x, send_local, counts = ops.dispatch(x, offsets, src_row, G)
        torch.cuda.synchronize()
        # bookkeeping, bit-exact: counts per owner rank, local ids, packed rows
        off = offsets.cpu().numpy()
        per = E // G
        assert counts.cpu().tolist() == [int(off[(h + 1) * per] - off[h * per]) for h in range(G)]
        expert = np.searchsorted(off, np.arange(len(src_row)), side="right") - 1
        assert np.array_equal(send_local.cpu().numpy(), expert % per)
        assert torch.equal(send_x.cpu(), xs[g][src_row.cpu().long() // k])
        state.append(dict(ids=ids, w=w, dst_of=dst_of, send_x=send_x, send_local=send_local,
                          counts=counts.cpu().tolist()))
    # the first all-to-all: rank h receives, from every rank g in order, g's rows for h
    y_recv = []
    for h in range(G):
        parts_x, parts_l = [], []
        for g in range(G):
            c = state[g]["counts"]
            a = sum(c[:h])
            parts_x.append(state[g]["send_x"][a:a + c[h]])
            parts_l.append(state[g]["send_local"][a:a + c[h]])
        y_recv.append(ops.expert_ffn(torch.cat(parts_x).contiguous(), torch.cat(parts_l).contiguous(), E // G,
                                     shards[h]))
    # the way back: rank g collects its rows from every h in order (its grouped order)
    ox = OracleExperts(cfg, seed)
    for g in range(G):
        parts = []
        for h in range(G):
            before = sum(state[q]["counts"][h] for q in range(g))  # rows of lower ranks in h's receive order
            parts.append(y_recv[h][before:before + state[g]["counts"][h]])
        y_back = torch.cat(parts).contiguous()
        y = ops.combine(y_back, state[g]["dst_of"], state[g]["w"]).cpu().numpy()
        ref = oracle.moe_layer(xs[g], bf16_bits(wg), None, ox, k, threads=THREADS)
        ids = state[g]["ids"].cpu().numpy()
        srt = -np.sort(-ref["logits"], axis=1)
        flagged = (srt[:, k - 1] - srt[:, k]) < 1e-3
        same = np.array([set(a) == set(b) for a, b in zip(ids, ref["ids"])])
        assert np.all(same | flagged)
        assert max_err_over_rms(y[same], ref["y"][same]) <= TOL_RMS


def test_ep_dispatch_of_no_tokens(mx):
    counts = torch.full((4,), -1, dtype=torch.int32, device=DEV)
    x = torch.empty((0, 256), dtype=torch.bfloat16, device=DEV)
    offsets = torch.zeros(17, dtype=torch.int32, device=DEV)
    src = torch.empty(0, dtype=torch.int32, device=DEV)
    mx.mxmoe_ep_dispatch(x, offsets, src, 2, 16, 4, torch.empty((0, 256), dtype=torch.bfloat16, device=DEV),
                         torch.empty(0, dtype=torch.int32, device=DEV), counts)
    assert counts.cpu().tolist() == [0, 0, 0, 0]
