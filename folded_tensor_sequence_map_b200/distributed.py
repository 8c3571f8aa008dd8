"""The folded layer's forward and backward on D processes, one rank each,
through ``torch.distributed`` ("Zyphra TSP folds TP+SP onto one GPU axis,
2.6x throughput on 1,024 MI300Xs", zubnet.ai, paragraphs 1-2).

Rank r holds its L = S/D tokens.  Forward: ``tsp_rank_forward_qkv`` (Q, and
its K/V rows at their global positions), the K/V all-gather, then
``tsp_rank_forward_out`` (attention over all keys, the out-projection, the
ring MLP).  Backward: ``tsp_rank_backward_attn`` (MLP, out-projection and
attention backward of the rank's rows, with its share of every key's dK/dV),
the dK/dV reduce-scatter to the keys' owners, ``tsp_rank_backward_qkv`` (QKV
projection and RMSNorm1 backward), then the all-reduce of the weight and
gain gradients.  Every step of the arithmetic runs in the library's kernels;
this module only moves tensors between the ranks.  The weights are whole on
every rank (the broadcast and ring schedules deliver every shard; their
order is the library's K-loop order).  With a backend other than NCCL the
exchanges go through host copies.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import tsp as T


def chunk_rows(plan: T.Plan, rank: int):
    """Global position ranges of rank `rank`'s tokens: its zigzag chunks
    rank and 2D-1-rank, c = S/(2D) rows each."""
    c = plan.S // (2 * plan.D)
    return (rank * c, (rank + 1) * c), ((2 * plan.D - 1 - rank) * c, (2 * plan.D - rank) * c)


def all_gather_kv(plan: T.Plan, rank: int, k: torch.Tensor, v: torch.Tensor, group=None) -> None:
    """Fill every rank's k, v ([S][h], global order) with all ranks' rows:
    two all-gathers of c-row blocks per tensor (each rank's low chunks, then
    its high chunks).  NCCL gathers into the device tensors directly; another
    backend goes through host copies."""
    D = plan.D
    on_device = dist.get_backend(group) == "nccl"
    for t in (k, v):
        for which in (0, 1):
            outs = [t[chunk_rows(plan, j)[which][0]:chunk_rows(plan, j)[which][1]] for j in range(D)]
            lo, hi = chunk_rows(plan, rank)[which]
            mine = t[lo:hi]
            if on_device:
                dist.all_gather(outs, mine.contiguous(), group=group)
            else:
                host = [torch.empty(o.shape, dtype=o.dtype) for o in outs]
                dist.all_gather(host, mine.cpu(), group=group)
                for o, hst in zip(outs, host):
                    o.copy_(hst)


def rank_forward(plan: T.Plan, rank: int, x, g1, wqkv, wo, g2, w1, w2, z, k, v, ws, group=None) -> None:
    """z = this rank's rows of the layer output, from this rank's tokens x."""
    T.tsp_rank_forward_qkv(plan, rank, x, g1, wqkv, k, v, ws)
    torch.cuda.current_stream().synchronize()
    all_gather_kv(plan, rank, k, v, group)
    T.tsp_rank_forward_out(plan, rank, x, k, v, wo, g2, w1, w2, z, ws)


def reduce_scatter_rows(plan: T.Plan, rank: int, part: torch.Tensor, out: torch.Tensor, group=None) -> None:
    """out ([L][h]) = the sum over the ranks of rows [rank L, (rank + 1) L) of
    their `part` ([S][h], rank-major local rows)."""
    L = plan.S // plan.D
    if dist.get_backend(group) == "nccl":
        dist.reduce_scatter_tensor(out, part, group=group)
    else:
        host = part.cpu()
        dist.all_reduce(host, group=group)
        out.copy_(host[rank * L:(rank + 1) * L])


def all_reduce_sum(tensors, group=None) -> None:
    """Sum each tensor over the ranks, in place."""
    on_device = dist.get_backend(group) == "nccl"
    for t in tensors:
        if on_device:
            dist.all_reduce(t, group=group)
        else:
            host = t.cpu()
            dist.all_reduce(host, group=group)
            t.copy_(host)


def rank_backward(plan: T.Plan, rank: int, dz, x, g1, g2, k, v, ws, bws, grads: dict, scratch: dict,
                  group=None) -> None:
    """Gradients of the layer from this rank's dz rows, after ``rank_forward``
    with the same ws, k, v.  grads: dx (bf16 [L][h], this rank's rows) and
    dg1, dwqkv, dwo, dg2, dw1, dw2 (fp32, summed over the ranks on return).
    scratch: dk_part, dv_part (fp32 [S][h]) and dk, dv (fp32 [L][h])."""
    g = grads
    T.tsp_rank_backward_attn(plan, rank, dz, k, v, g2, ws, bws, scratch["dk_part"], scratch["dv_part"], g["dwo"],
                             g["dg2"], g["dw1"], g["dw2"])
    torch.cuda.current_stream().synchronize()
    reduce_scatter_rows(plan, rank, scratch["dk_part"], scratch["dk"], group)
    reduce_scatter_rows(plan, rank, scratch["dv_part"], scratch["dv"], group)
    T.tsp_rank_backward_qkv(plan, rank, x, g1, scratch["dk"], scratch["dv"], ws, bws, g["dx"], g["dg1"], g["dwqkv"])
    torch.cuda.current_stream().synchronize()
    all_reduce_sum([g[n] for n in ("dg1", "dwqkv", "dwo", "dg2", "dw1", "dw2")], group)
