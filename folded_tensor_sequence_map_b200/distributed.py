"""The folded layer's forward on D processes, one rank each, through
``torch.distributed`` ("Zyphra TSP folds TP+SP onto one GPU axis, 2.6x
throughput on 1,024 MI300Xs", zubnet.ai, paragraphs 1-2).

Rank r holds its L = S/D tokens and runs ``tsp_rank_forward_qkv`` (Q, and
its K/V rows at their global positions), the K/V all-gather, then
``tsp_rank_forward_out`` (attention over all keys, the out-projection, the
ring MLP).  Every step of the arithmetic runs in the library's kernels; this
module only moves K and V between the ranks.  The weights are whole on every
rank (the broadcast and ring schedules deliver every shard; their order is
the library's K-loop order).
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
