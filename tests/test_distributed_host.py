"""The exchanges of ``folded_tensor_sequence_map_b200.distributed`` on two
gloo ranks on CPU (the host-staging branch, which moves the same rows as the
NCCL one): which rows each rank contributes and receives in the K/V
all-gather, the dK/dV reduce-scatter and the gradient all-reduce.  The
layout they must reproduce is the zigzag partition ("Zyphra TSP folds TP+SP
onto one GPU axis, 2.6x throughput on 1,024 MI300Xs", zubnet.ai, paragraph
2), taken here from the oracle's map."""

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O

H_COLS = 8
SHAPE = dict(h=128, heads=4, ffn=512, S=1024, D=2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import folded_tensor_sequence_map_b200 as T
    import folded_tensor_sequence_map_b200.distributed as TD

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        s = SHAPE
        plan = T.tsp_plan(s["h"], s["heads"], s["ffn"], s["S"], s["D"])
        S, L = s["S"], s["S"] // s["D"]
        zig = O.zigzag_map(S, s["D"]).ravel()
        # K/V all-gather: each rank writes only its own tokens' rows (global
        # positions zig[rank L .. (rank + 1) L)), value = position + 1
        k = torch.zeros(S, H_COLS, dtype=torch.float16)
        v = torch.zeros(S, H_COLS, dtype=torch.float16)
        pos = torch.from_numpy(zig[rank * L:(rank + 1) * L].astype(np.int64))
        k[pos] = (pos.to(torch.float16) + 1).unsqueeze(1).expand(-1, H_COLS)
        v[pos] = -(pos.to(torch.float16) + 1).unsqueeze(1).expand(-1, H_COLS)
        TD.all_gather_kv(plan, rank, k, v)
        # dK/dV reduce-scatter: rank r's partial rows are (r + 1) * (row + 1);
        # rank r receives the sum over ranks of rows [r L, (r + 1) L)
        part = (torch.arange(S, dtype=torch.float32) + 1).unsqueeze(1).repeat(1, H_COLS) * (rank + 1)
        got = torch.empty(L, H_COLS)
        TD.reduce_scatter_rows(plan, rank, part, got)
        # gradient all-reduce
        g = torch.full((3, 5), float(rank + 1))
        TD.all_reduce_sum([g])
        out[rank] = (k.float().numpy(), v.float().numpy(), got.numpy(), g.numpy())
    finally:
        dist.destroy_process_group()


def test_exchanges_move_the_zigzag_rows():
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    S, L, D = SHAPE["S"], SHAPE["S"] // SHAPE["D"], SHAPE["D"]
    full = np.repeat((np.arange(S, dtype=np.float32) + 1)[:, None], H_COLS, axis=1)
    for r in range(D):
        k, v, got, g = out[r]
        # every rank holds every position's row after the all-gather
        assert np.array_equal(k, full) and np.array_equal(v, -full), r
        # rows [r L, (r + 1) L), summed over the ranks' factors 1 + 2
        assert np.array_equal(got, full[r * L:(r + 1) * L] * 3), r
        assert np.array_equal(g, np.full((3, 5), 3.0)), r


def test_chunk_rows_are_the_oracle_zigzag_chunks():
    import folded_tensor_sequence_map_b200 as T
    import folded_tensor_sequence_map_b200.distributed as TD

    for h, heads, ffn, S, D in ((128, 4, 512, 1024, 2), (128, 4, 512, 2048, 4), (256, 8, 1024, 32768, 8)):
        plan = T.tsp_plan(h, heads, ffn, S, D)
        zig = O.zigzag_map(S, D).ravel()
        L = S // D
        for r in range(D):
            (a0, a1), (b0, b1) = TD.chunk_rows(plan, r)
            want = np.concatenate([np.arange(a0, a1), np.arange(b0, b1)])
            assert np.array_equal(zig[r * L:(r + 1) * L], want), (S, D, r)
