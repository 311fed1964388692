"""The expert-parallel layer's partition and exchange logic on CPU: two (and
three) gloo ranks run mxfp4_quantized_moe_router_b200.ep.layer_forward_ep with
its compute steps replaced by the float64 oracle, and each rank's output must
equal the oracle's whole layer (all experts in one process) on that rank's
tokens. Only the exchanges (all_to_all_single with uneven splits, forward and
back) and the bookkeeping around them are under test here; the GPU kernels of
the same steps are checked in tests/test_gpu_ep.py.

Page: the SGLang launch in the "MiMo-V2.5-Pro-FP4-DFlash" model card's
deployment section serves the model with --ep-size 16.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_WORKER = r"""
import json, os, sys
sys.path.insert(0, sys.argv[1])
import numpy as np
import torch
import torch.distributed as dist
import datagen
import oracle
from mxfp4_quantized_moe_router_b200 import ep

def bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)

class OracleOps:
    # the layer's compute steps in float64 on the host (a test double of ep.LibOps)
    def __init__(self, cfg, experts):
        self.cfg, self.experts = cfg, experts
    def route(self, x, wg, bias):
        ids, w = oracle.route(oracle.router_logits(bits(x), bits(wg), bias), self.cfg.k)
        return torch.from_numpy(ids), torch.from_numpy(w)
    def group(self, ids):
        off, src, dst = oracle.permute(ids.numpy(), self.cfg.E)
        return torch.from_numpy(off), torch.from_numpy(src), torch.from_numpy(dst)
    def dispatch(self, x, offsets, src_row, G):
        per = self.cfg.E // G
        off = offsets.numpy()
        expert = np.searchsorted(off, np.arange(len(src_row)), side="right") - 1
        send_x = x[src_row.long() // self.cfg.k]
        send_local = torch.from_numpy((expert % per).astype(np.int32))
        counts = torch.tensor([off[(g + 1) * per] - off[g * per] for g in range(G)], dtype=torch.int32)
        return send_x, send_local, counts
    def expert_ffn(self, x_recv, recv_local, E_local, prepacked_local):
        y = np.zeros((x_recv.shape[0], self.cfg.H))
        xb = bits(x_recv)
        for e in range(E_local):
            rows = np.nonzero(recv_local.numpy() == e)[0]
            if len(rows):
                y[rows] = oracle.expert_ffn_mxfp4(*prepacked_local[e], np.ascontiguousarray(xb[rows]))
        return torch.from_numpy(y)
    def combine(self, y_back, dst_of, w):
        T, k = w.shape
        return torch.from_numpy(oracle.combine(y_back.numpy(), dst_of.numpy(), w.numpy(), T, k))

world = int(os.environ["WORLD_SIZE"]); rank = int(os.environ["RANK"])
dist.init_process_group("gloo", init_method="env://", world_size=world, rank=rank)
cfg = datagen.LayerConfig("ep", 128, 12, 3, 64, 5 + 4 * rank)   # ranks hold different token counts
experts = {}
for e in range(cfg.E):
    experts[e] = oracle.quantize(datagen.make_w13(cfg, e, 0)) + oracle.quantize(datagen.make_w2(cfg, e, 0))
e0, e1 = ep.expert_range(cfg.E, world, rank)
local = [experts[e] for e in range(e0, e1)]
x = datagen.make_x(cfg, 100 + rank)
wg = datagen.make_router_weight(cfg, 0)
y, ids, w = ep.layer_forward_ep(x, wg, None, local, cfg.E, cfg.I, cfg.k, ops=OracleOps(cfg, experts))
ref = oracle.moe_layer(x, wg, None, lambda e: experts[e], cfg.k)
dist.destroy_process_group()
print(json.dumps({"rank": rank, "ids_equal": bool(np.array_equal(ids.numpy(), ref["ids"])),
                  "max_abs_err": float(np.max(np.abs(y.numpy() - ref["y"]))), "rms": float(np.sqrt(np.mean(ref["y"] ** 2))),
                  "range": [e0, e1]}))
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_ep_layer_matches_the_whole_layer_on_gloo_ranks(world):
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, WORLD_SIZE=str(world), RANK=str(r), LOCAL_RANK=str(r), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", _WORKER, ROOT], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True, cwd=ROOT))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=300)
        assert p.returncode == 0, err[-3000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    per = 12 // world
    for o in outs:
        assert o["range"] == [o["rank"] * per, (o["rank"] + 1) * per]
        assert o["ids_equal"]
        # the same float64 steps on both sides, only moved between ranks: equal to rounding
        assert o["max_abs_err"] <= 1e-12 * max(o["rms"], 1e-30)


def test_expert_range_splits_evenly():
    sys.path.insert(0, ROOT)
    from mxfp4_quantized_moe_router_b200 import ep

    assert [ep.expert_range(384, 16, g) for g in (0, 1, 15)] == [(0, 24), (24, 48), (360, 384)]
    with pytest.raises(ValueError):
        ep.expert_range(384, 7, 0)
