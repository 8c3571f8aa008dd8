"""The method's collectives on D real processes (torch.distributed, gloo, CPU).

"Zyphra TSP folds TP+SP onto one GPU axis, 2.6x throughput on 1,024 MI300Xs"
(zubnet.ai), paragraphs 1-2: each of D ranks keeps 1/D of the weights and 1/D
of the tokens; attention weight shards are broadcast one after another and
applied by every rank to its own tokens, K/V are all-gathered under the zigzag
partition, and the MLP weight shards travel a ring whose partial sums stay on
their rank.  The backward runs the reverse: weight-gradient pieces are reduced
to the shard's owner, key/value gradients are summed over every rank's
queries and kept at the key's owner.

Here every rank is a separate process that holds only its own tokens and its
own weight shards and obtains every other shard through the collective the
schedule names (dist.broadcast, dist.all_gather, dist.isend/irecv around the
ring, dist.reduce to the owner, dist.all_reduce).  Per-rank arithmetic uses
the oracle's fp64 primitives.  The test checks, for D = 2 and 4 on the tiny
layer:
* the shards each rank applied, step by step, equal the oracle's schedules
  bit for bit (broadcast: shard t at step t; ring: shard (r + t) mod D);
* each rank's z and dx rows and each owner's weight-gradient shard equal the
  oracle's folded layer (simulated ranks in one process) to fp64 rounding.
"""

import datetime
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from synth_inputs import LayerShape, bits_to_f32, make_layer_inputs

SHAPE = dict(h=128, heads=4, ffn=512, S=256)
SEED = 0


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _t(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))


def _weights(inp):
    w = {k: bits_to_f32(inp[k]).astype(np.float64) for k in ("wqkv", "wo", "w1", "w2")}
    w["g1"] = inp["g1"].astype(np.float64)
    w["g2"] = inp["g2"].astype(np.float64)
    return w


def _ring_pass(bufs, rank, D):
    """After a ring step rank r holds what rank r+1 held: send to r-1, receive
    from r+1 (every buffer of the shard, in order)."""
    out = [torch.empty_like(b) for b in bufs]
    reqs = []
    for b, o in zip(bufs, out):
        reqs.append(dist.isend(b, (rank - 1) % D))
        reqs.append(dist.irecv(o, (rank + 1) % D))
    for r in reqs:
        r.wait()
    return out


def _rank_main(rank, D, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=D, timeout=datetime.timedelta(seconds=120))
    try:
        _run_rank(rank, D, out_dir)
    finally:
        dist.destroy_process_group()


def _run_rank(rank, D, out_dir):
    shape = LayerShape(D=D, **SHAPE)
    h, H, F, S = shape.h, shape.heads, shape.ffn, shape.S
    dh, L = h // H, S // D
    inp = make_layer_inputs(shape, SEED)
    W = _weights(inp)
    zig = O.zigzag_map(S, D)
    hp = H // D
    cols = lambda t: O.head_cols(t, H, D, dh)
    units = lambda s: O.ffn_units(s, F, D)
    # what this rank owns: its tokens and its shards (nothing else is read below)
    x = bits_to_f32(inp["x"][zig[rank]]).astype(np.float64)
    dz = bits_to_f32(inp["dy"][zig[rank]]).astype(np.float64)
    c = cols(rank)
    own_qkv = np.concatenate([W["wqkv"][j * h:(j + 1) * h][c] for j in range(3)])  # [3 hp dh, h]
    own_wo = np.ascontiguousarray(W["wo"][:, c])                                  # [h, hp dh]
    own_w1 = np.ascontiguousarray(W["w1"][units(rank)])                           # [F/D, h]
    own_w2 = np.ascontiguousarray(W["w2"][:, units(rank)])                        # [h, F/D]
    g1, g2 = W["g1"], W["g2"]
    del W, inp

    def bcast(own, t):
        buf = _t(own) if rank == t else torch.empty(own.shape, dtype=torch.float64)
        dist.broadcast(buf, src=t)
        return buf.numpy()

    bcast_log, ring_log = [], []
    # ---- forward
    a, rstd1 = O.rmsnorm(x, g1)
    Q, K, V = np.zeros((L, h)), np.zeros((L, h)), np.zeros((L, h))
    for t in range(D):
        sh = bcast(own_qkv, t)
        bcast_log.append(t)
        n = hp * dh
        Q[:, cols(t)] = a @ sh[:n].T
        K[:, cols(t)] = a @ sh[n:2 * n].T
        V[:, cols(t)] = a @ sh[2 * n:].T
    Kg, Vg = np.zeros((S, h)), np.zeros((S, h))
    for src, dst in ((K, Kg), (V, Vg)):
        parts = [torch.empty(L, h, dtype=torch.float64) for _ in range(D)]
        dist.all_gather(parts, _t(src))
        for j in range(D):
            dst[zig[j]] = parts[j].numpy()
    Ob, lse = O.causal_attention(Q, Kg, Vg, zig[rank], H)
    acc = np.zeros((L, h))
    for t in range(D):
        acc += Ob[:, cols(t)] @ bcast(own_wo, t).T
    y = x + acc
    b, rstd2 = O.rmsnorm(y, g2)
    U = np.zeros((L, F))
    acc = np.zeros((L, h))
    cur = [_t(own_w1), _t(own_w2), torch.tensor([rank])]
    for t in range(D):
        s = int(cur[2].item())
        ring_log.append(s)
        u = b @ cur[0].numpy().T
        U[:, units(s)] = u
        acc += O.gelu_tanh(u) @ cur[1].numpy().T
        if t + 1 < D:
            cur = _ring_pass(cur, rank, D)
    z = y + acc

    # ---- backward
    pieces_w1, pieces_w2 = {}, {}
    db = np.zeros((L, h))
    cur = [_t(own_w1), _t(own_w2), torch.tensor([rank])]
    for t in range(D):
        s = int(cur[2].item())
        u = U[:, units(s)]
        du = (dz @ cur[1].numpy()) * O.gelu_tanh_grad(u)
        pieces_w2[s] = dz.T @ O.gelu_tanh(u)
        pieces_w1[s] = du.T @ b
        db += du @ cur[0].numpy()
        if t + 1 < D:
            cur = _ring_pass(cur, rank, D)
    # weight-gradient pieces reduced to each shard's owner (rank order of the
    # calls is the same on every rank)
    mine = {}
    for s in range(D):
        for name, p in (("dw1", pieces_w1[s]), ("dw2", pieces_w2[s])):
            buf = _t(p)
            dist.reduce(buf, dst=s, op=dist.ReduceOp.SUM)
            if rank == s:
                mine[name] = buf.numpy().copy()
    dyn, dg2 = O.rmsnorm_backward(db, y, rstd2, g2)
    dy = dz + dyn
    dO = np.zeros((L, h))
    for t in range(D):
        dO[:, cols(t)] = dy @ bcast(own_wo, t)
        buf = _t(dy.T @ Ob[:, cols(t)])
        dist.reduce(buf, dst=t, op=dist.ReduceOp.SUM)
        if rank == t:
            mine["dwo"] = buf.numpy().copy()
    dq, dkg, dvg = O.causal_attention_backward(Q, Kg, Vg, Ob, dO, lse, zig[rank], H)
    # key/value gradients: summed over every rank's queries, kept at the owner
    dK, dV = None, None
    for g, name in ((dkg, "dk"), (dvg, "dv")):
        buf = _t(g)
        dist.all_reduce(buf, op=dist.ReduceOp.SUM)
        rows = buf.numpy()[zig[rank]]
        if name == "dk":
            dK = rows
        else:
            dV = rows
    da = np.zeros((L, h))
    n = hp * dh
    for t in range(D):
        sh = bcast(own_qkv, t)
        c = cols(t)
        da += dq[:, c] @ sh[:n] + dK[:, c] @ sh[n:2 * n] + dV[:, c] @ sh[2 * n:]
        buf = _t(np.concatenate([dq[:, c].T @ a, dK[:, c].T @ a, dV[:, c].T @ a]))
        dist.reduce(buf, dst=t, op=dist.ReduceOp.SUM)
        if rank == t:
            mine["dwqkv"] = buf.numpy().copy()
    dxn, dg1 = O.rmsnorm_backward(da, x, rstd1, g1)
    dx = dy + dxn
    for g in (dg1, dg2):
        buf = _t(g)
        dist.all_reduce(buf, op=dist.ReduceOp.SUM)
        g[:] = buf.numpy()
    np.savez(os.path.join(out_dir, f"rank{rank}.npz"), z=z, dx=dx, dg1=dg1, dg2=dg2,
             bcast=np.array(bcast_log), ring=np.array(ring_log), **mine)


@pytest.mark.parametrize("D", [2, 4])
def test_collectives_match_the_oracle(D):
    shape = LayerShape(D=D, **SHAPE)
    h, H, F, S = shape.h, shape.heads, shape.ffn, shape.S
    dh, L = h // H, S // D
    with tempfile.TemporaryDirectory() as out_dir:
        mp.start_processes(_rank_main, args=(D, _free_port(), out_dir), nprocs=D, join=True, start_method="spawn")
        res = [dict(np.load(os.path.join(out_dir, f"rank{r}.npz"))) for r in range(D)]
    inp = make_layer_inputs(shape, SEED)
    w = _weights(inp)
    zig = O.zigzag_map(S, D).ravel()
    zo, cache = O.tsp_layer_forward(bits_to_f32(inp["x"][zig]).astype(np.float64), w, H, D)
    go = O.tsp_layer_backward(bits_to_f32(inp["dy"][zig]).astype(np.float64), w, cache)
    bsched, rsched = O.shard_schedule(D, 0), O.shard_schedule(D, 1)

    def close(a, b, name):
        err = np.max(np.abs(a - b)) / np.max(np.abs(b))
        assert err < 1e-10, (name, err)

    for r in range(D):
        rr = res[r]
        assert np.array_equal(rr["bcast"], bsched[:, r]), r
        assert np.array_equal(rr["ring"], rsched[:, r]), r
        close(rr["z"], zo[r * L:(r + 1) * L], "z")
        close(rr["dx"], go["dx"][r * L:(r + 1) * L], "dx")
        close(rr["dg1"], go["dg1"], "dg1")
        close(rr["dg2"], go["dg2"], "dg2")
        c = O.head_cols(r, H, D, dh)
        u = O.ffn_units(r, F, D)
        close(rr["dwqkv"], np.concatenate([go["dwqkv"][j * h:(j + 1) * h][c] for j in range(3)]), "dwqkv")
        close(rr["dwo"], go["dwo"][:, c], "dwo")
        close(rr["dw1"], go["dw1"][u], "dw1")
        close(rr["dw2"], go["dw2"][:, u], "dw2")
