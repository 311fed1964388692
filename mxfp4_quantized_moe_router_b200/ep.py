"""Expert-parallel MoE layer: the 384 experts split over the ranks of a
torch.distributed group, each rank routing its own tokens.

The pages serve the model with expert parallelism (--ep-size 16 in the SGLang
launch of the "MiMo-V2.5-Pro-FP4-DFlash" model card's deployment section and
the nxbn.cn article's SGLang deployment section). Rank g of G holds experts
[g E/G, (g+1) E/G) as its own prepacked blob. One step (include/mxmoe.h,
"Expert parallelism"):

  router + route on the rank's tokens -> group pairs by expert (= by owner
  rank) -> pack rows, local expert ids and per-rank counts -> all-to-all of
  counts, rows and ids -> the rank's experts on what it received -> all-to-all
  back (reverse splits) -> weighted combine in slot order.

Every compute step runs in libmxmoe's kernels through the C ABI (``LibOps``);
this module only moves buffers with torch.distributed's all_to_all_single
(NCCL over NVLink on GPUs). The split sizes cross to the host once per step
(the counts' all-to-all), as NCCL's all-to-all with uneven splits needs them.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

import mxfp4_quantized_moe_router_b200 as mx


def expert_range(E: int, G: int, rank: int) -> tuple[int, int]:
    """The contiguous experts [e0, e1) that rank `rank` of G holds."""
    if E % G:
        raise ValueError("E=%d is not a multiple of the group size %d" % (E, G))
    per = E // G
    return rank * per, (rank + 1) * per


class LibOps:
    """The layer's compute steps on the device, each one C-ABI call."""

    def __init__(self, H: int, I: int, E: int, k: int):
        self.H, self.I, self.E, self.k = H, I, E, k

    def route(self, x, wg, bias):
        T = x.shape[0]
        dev = x.device
        logits = torch.empty((T, self.E), dtype=torch.float32, device=dev)
        ids = torch.empty((T, self.k), dtype=torch.int32, device=dev)
        w = torch.empty((T, self.k), dtype=torch.float32, device=dev)
        mx.mxmoe_router_gemm(x, wg, bias, logits)
        mx.mxmoe_route(logits, self.k, ids, w)
        return ids, w

    def group(self, ids):
        T, k = ids.shape
        dev = ids.device
        offsets = torch.empty(self.E + 1, dtype=torch.int32, device=dev)
        src_row = torch.empty(T * k, dtype=torch.int32, device=dev)
        dst_of = torch.empty(T * k, dtype=torch.int32, device=dev)
        scratch = torch.empty(max(1, mx.mxmoe_permute_scratch_size(T, k, self.E)), dtype=torch.uint8, device=dev)
        mx.mxmoe_permute_ws(ids, self.E, offsets, src_row, dst_of, scratch)
        return offsets, src_row, dst_of

    def dispatch(self, x, offsets, src_row, G):
        T, H = x.shape
        n = T * self.k
        send_x = torch.empty((n, H), dtype=torch.bfloat16, device=x.device)
        send_local = torch.empty(n, dtype=torch.int32, device=x.device)
        send_counts = torch.empty(G, dtype=torch.int32, device=x.device)
        mx.mxmoe_ep_dispatch(x, offsets, src_row, self.k, self.E, G, send_x, send_local, send_counts)
        return send_x, send_local, send_counts

    def expert_ffn(self, x_recv, recv_local, E_local, prepacked_local):
        n, H = x_recv.shape
        y = torch.empty((n, H), dtype=torch.float32, device=x_recv.device)
        ws = torch.empty(max(1, mx.mxmoe_ep_workspace_size(n, E_local, H, self.I)), dtype=torch.uint8,
                         device=x_recv.device)
        mx.mxmoe_ep_expert_ffn(x_recv, recv_local, E_local, self.I, prepacked_local, y, ws)
        return y

    def combine(self, y_back, dst_of, w):
        T, k = w.shape
        y = torch.empty((T, self.H), dtype=torch.float32, device=w.device)
        mx.mxmoe_combine(y_back, dst_of, w, y)
        return y


def layer_forward_ep(x, wg, bias, prepacked_local, E: int, I: int, k: int, group=None, ops=None):
    """The MoE layer on this rank's tokens x (bf16 [T, H]) with the experts
    split over `group`; prepacked_local holds this rank's experts
    (expert_range). Returns (y float32 [T, H], ids int32 [T, k], w float32
    [T, k]). Every rank of the group must call it, in the same order."""
    G = dist.get_world_size(group)
    T, H = x.shape
    ops = ops if ops is not None else LibOps(H, I, E, k)
    E_local = E // G
    expert_range(E, G, 0)  # E must split evenly
    ids, w = ops.route(x, wg, bias)
    offsets, src_row, dst_of = ops.group(ids)
    send_x, send_local, send_counts = ops.dispatch(x, offsets, src_row, G)
    recv_counts = torch.empty_like(send_counts)
    dist.all_to_all_single(recv_counts, send_counts, group=group)
    sc = [int(v) for v in send_counts.tolist()]
    rc = [int(v) for v in recv_counts.tolist()]
    n_recv = sum(rc)
    x_recv = torch.empty((n_recv, H), dtype=send_x.dtype, device=send_x.device)
    recv_local = torch.empty(n_recv, dtype=torch.int32, device=send_x.device)
    dist.all_to_all_single(x_recv, send_x, rc, sc, group=group)
    dist.all_to_all_single(recv_local, send_local, rc, sc, group=group)
    y_recv = ops.expert_ffn(x_recv, recv_local, E_local, prepacked_local)
    y_back = torch.empty((T * k, H), dtype=y_recv.dtype, device=y_recv.device)
    dist.all_to_all_single(y_back, y_recv, sc, rc, group=group)
    return ops.combine(y_back, dst_of, w), ids, w
