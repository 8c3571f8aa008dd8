"""One rank's share of the forward (``tsp_rank_forward_qkv`` / ``_out``) and
of the backward (``tsp_rank_backward_attn`` / ``_qkv``), the entry points for
running the folded layer on D devices ("Zyphra TSP folds TP+SP onto one GPU
axis, 2.6x throughput on 1,024 MI300Xs", zubnet.ai, paragraphs 1-2).

* On one device, the D ranks run in turn over shared K/V buffers (the
  all-gather then needs no copy): every rank's z rows, and the K/V they
  write, are bit for bit those of ``tsp_layer_forward`` (the same kernels on
  the same rows), for the tiny width with D = 2 and 4 and the 7B layer at
  S=4096, D=8.
* Two processes, one rank each, exchange K/V with torch.distributed (gloo,
  through host copies) as ``folded_tensor_sequence_map_b200.distributed``
  does on D GPUs; their z rows are again the layer's.  Both processes use the
  one GPU here; the kernels of one never wait on the other's.
* Backward (head size 128): the D ranks in turn, with the dK/dV partial sums
  and the weight gradients summed on the device between the calls as the
  reduce-scatter and all-reduce would, give every gradient within the stated
  bounds of the fp64 oracle; and two processes do the same through
  ``distributed.rank_backward`` (gloo).
"""

import os
import socket
import tempfile

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import folded_tensor_sequence_map_b200 as T
import oracle as O
from synth_inputs import LayerShape, bits_to_f32, make_layer_inputs
from tests.gpu_helpers import GpuLayer, assert_close, dev_bf16, host_f64, oracle_weights

SHAPES = [
    (LayerShape(h=128, heads=4, ffn=512, S=1024, D=2), 11),
    (LayerShape(h=128, heads=4, ffn=512, S=2048, D=4), 12),
    (LayerShape(h=4096, heads=32, ffn=16384, S=4096, D=8), 13),
]


def _layer(shape, inp):
    layer = GpuLayer(shape, inp, training=True)
    z = layer.forward().clone()
    k = layer.saved_view("k", (shape.S, shape.h), torch.float16).clone()
    v = layer.saved_view("v", (shape.S, shape.h), torch.float16).clone()
    return layer, z, k, v


@pytest.mark.parametrize("shape,seed", SHAPES, ids=["tiny_d2", "tiny_d4", "7b_s4096_d8"])
def test_ranks_in_turn_equal_the_layer(shape, seed):
    inp = make_layer_inputs(shape, seed, with_dy=False)
    layer, z_ref, k_ref, v_ref = _layer(shape, inp)
    s, L = shape, shape.S // shape.D
    plan = layer.plan
    x = layer.x
    w = layer.w
    k = torch.zeros(s.S, s.h, dtype=torch.float16, device="cuda")
    v = torch.zeros_like(k)
    wss = [torch.empty(T.tsp_rank_workspace_size(plan), dtype=torch.uint8, device="cuda") for _ in range(s.D)]
    for r in range(s.D):
        T.tsp_rank_forward_qkv(plan, r, x[r * L:(r + 1) * L], layer.g1, w["wqkv"], k, v, wss[r])
    T.tsp_sync_status(plan)
    assert torch.equal(k, k_ref) and torch.equal(v, v_ref)
    z = torch.empty_like(z_ref)
    for r in range(s.D):
        T.tsp_rank_forward_out(plan, r, x[r * L:(r + 1) * L], k, v, w["wo"], layer.g2, w["w1"], w["w2"],
                               z[r * L:(r + 1) * L], wss[r])
    T.tsp_sync_status(plan)
    assert torch.equal(z, z_ref)


def _free_port():
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def _rank_main(rank, world, port, out_dir, shape_args, seed):
    import torch.distributed as dist

    import folded_tensor_sequence_map_b200.distributed as TD

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        shape = LayerShape(**shape_args)
        inp = make_layer_inputs(shape, seed, with_dy=False)
        plan = T.tsp_plan(shape.h, shape.heads, shape.ffn, shape.S, shape.D)
        zig = T.tsp_zigzag_map(plan)
        L = shape.S // shape.D
        x = dev_bf16(inp["x"][zig][rank * L:(rank + 1) * L])          # this rank's tokens only
        w = {kk: dev_bf16(inp[kk]) for kk in ("wqkv", "wo", "w1", "w2")}
        g1 = torch.from_numpy(inp["g1"]).cuda()
        g2 = torch.from_numpy(inp["g2"]).cuda()
        k = torch.zeros(shape.S, shape.h, dtype=torch.float16, device="cuda")
        v = torch.zeros_like(k)
        ws = torch.empty(T.tsp_rank_workspace_size(plan), dtype=torch.uint8, device="cuda")
        z = torch.empty(L, shape.h, dtype=torch.bfloat16, device="cuda")
        TD.rank_forward(plan, rank, x, g1, w["wqkv"], w["wo"], g2, w["w1"], w["w2"], z, k, v, ws)
        T.tsp_sync_status(plan)
        np.save(os.path.join(out_dir, f"z{rank}.npy"), z.view(torch.int16).cpu().numpy())
    finally:
        dist.destroy_process_group()


def test_two_processes_exchange_kv_and_equal_the_layer():
    import torch.multiprocessing as mp

    shape, seed = SHAPES[0]
    with tempfile.TemporaryDirectory() as out_dir:
        mp.start_processes(_rank_main, args=(shape.D, _free_port(), out_dir, vars(shape), seed), nprocs=shape.D,
                           join=True, start_method="spawn")
        zs = [np.load(os.path.join(out_dir, f"z{r}.npy")) for r in range(shape.D)]
    inp = make_layer_inputs(shape, seed, with_dy=False)
    _, z_ref, _, _ = _layer(shape, inp)
    assert np.array_equal(np.concatenate(zs), z_ref.view(torch.int16).cpu().numpy())


# ---- backward -----------------------------------------------------------------

BWD_SHAPES = [
    (LayerShape(h=256, heads=2, ffn=1024, S=1024, D=2), 21),
    (LayerShape(h=512, heads=4, ffn=2048, S=2048, D=4), 22),
    (LayerShape(h=4096, heads=32, ffn=16384, S=4096, D=8), 23),
]
GRADS = ("dg1", "dwqkv", "dwo", "dg2", "dw1", "dw2")


def _oracle_grads(shape, inp):
    zig = O.zigzag_map(shape.S, shape.D).ravel()
    w = oracle_weights(inp)
    zo, cache = O.tsp_layer_forward(bits_to_f32(inp["x"][zig]).astype(np.float64), w, shape.heads, shape.D)
    return zo, O.tsp_layer_backward(bits_to_f32(inp["dy"][zig]).astype(np.float64), w, cache)


def _grad_buffers(s, L):
    f32 = dict(dtype=torch.float32, device="cuda")
    return dict(dx=torch.empty(L, s.h, dtype=torch.bfloat16, device="cuda"), dg1=torch.empty(s.h, **f32),
                dwqkv=torch.empty(3 * s.h, s.h, **f32), dwo=torch.empty(s.h, s.h, **f32), dg2=torch.empty(s.h, **f32),
                dw1=torch.empty(s.ffn, s.h, **f32), dw2=torch.empty(s.h, s.ffn, **f32))


@pytest.mark.parametrize("shape,seed", BWD_SHAPES, ids=["h256_d2", "h512_d4", "7b_s4096_d8"])
def test_rank_backward_in_turn_against_oracle(shape, seed):
    s, L = shape, shape.S // shape.D
    inp = make_layer_inputs(shape, seed)
    plan = T.tsp_plan(s.h, s.heads, s.ffn, s.S, s.D)
    zig = T.tsp_zigzag_map(plan)
    x, dy = dev_bf16(inp["x"][zig]), dev_bf16(inp["dy"][zig])
    w = {kk: dev_bf16(inp[kk]) for kk in ("wqkv", "wo", "w1", "w2")}
    g1, g2 = torch.from_numpy(inp["g1"]).cuda(), torch.from_numpy(inp["g2"]).cuda()
    k = torch.zeros(s.S, s.h, dtype=torch.float16, device="cuda")
    v = torch.zeros_like(k)
    wss = [torch.empty(T.tsp_rank_workspace_size(plan), dtype=torch.uint8, device="cuda") for _ in range(s.D)]
    bws = [torch.empty(T.tsp_rank_backward_workspace_size(plan), dtype=torch.uint8, device="cuda")
           for _ in range(s.D)]
    rows = [slice(r * L, (r + 1) * L) for r in range(s.D)]
    for r in range(s.D):
        T.tsp_rank_forward_qkv(plan, r, x[rows[r]], g1, w["wqkv"], k, v, wss[r])
    z = torch.empty(s.S, s.h, dtype=torch.bfloat16, device="cuda")
    for r in range(s.D):
        T.tsp_rank_forward_out(plan, r, x[rows[r]], k, v, w["wo"], g2, w["w1"], w["w2"], z[rows[r]], wss[r])
    # attention side of every rank; the partial dK/dV summed as the
    # reduce-scatter would
    dk_part = torch.empty(s.S, s.h, dtype=torch.float32, device="cuda")
    dv_part = torch.empty_like(dk_part)
    dk_sum, dv_sum = torch.zeros_like(dk_part), torch.zeros_like(dk_part)
    per_rank = [_grad_buffers(s, L) for _ in range(s.D)]
    for r in range(s.D):
        g = per_rank[r]
        T.tsp_rank_backward_attn(plan, r, dy[rows[r]], k, v, g2, wss[r], bws[r], dk_part, dv_part, g["dwo"],
                                 g["dg2"], g["dw1"], g["dw2"])
        dk_sum += dk_part
        dv_sum += dv_part
    for r in range(s.D):
        g = per_rank[r]
        T.tsp_rank_backward_qkv(plan, r, x[rows[r]], g1, dk_sum[rows[r]].contiguous(), dv_sum[rows[r]].contiguous(),
                                wss[r], bws[r], g["dx"], g["dg1"], g["dwqkv"])
    T.tsp_sync_status(plan)
    got = {n: host_f64(sum(per_rank[r][n] for r in range(s.D))) for n in GRADS}
    got["dx"] = host_f64(torch.cat([per_rank[r]["dx"] for r in range(s.D)]))
    zo, go = _oracle_grads(shape, inp)
    assert_close("z", host_f64(z), zo)
    for n in ("dx",) + GRADS:
        assert_close(n, got[n], go[n])


def _rank_bwd_main(rank, world, port, out_dir, shape_args, seed):
    import torch.distributed as dist

    import folded_tensor_sequence_map_b200.distributed as TD

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        shape = LayerShape(**shape_args)
        s, L = shape, shape.S // shape.D
        inp = make_layer_inputs(shape, seed)
        plan = T.tsp_plan(s.h, s.heads, s.ffn, s.S, s.D)
        zig = T.tsp_zigzag_map(plan)
        mine = slice(rank * L, (rank + 1) * L)
        x, dz = dev_bf16(inp["x"][zig][mine]), dev_bf16(inp["dy"][zig][mine])
        w = {kk: dev_bf16(inp[kk]) for kk in ("wqkv", "wo", "w1", "w2")}
        g1, g2 = torch.from_numpy(inp["g1"]).cuda(), torch.from_numpy(inp["g2"]).cuda()
        k = torch.zeros(s.S, s.h, dtype=torch.float16, device="cuda")
        v = torch.zeros_like(k)
        ws = torch.empty(T.tsp_rank_workspace_size(plan), dtype=torch.uint8, device="cuda")
        bws = torch.empty(T.tsp_rank_backward_workspace_size(plan), dtype=torch.uint8, device="cuda")
        z = torch.empty(L, s.h, dtype=torch.bfloat16, device="cuda")
        TD.rank_forward(plan, rank, x, g1, w["wqkv"], w["wo"], g2, w["w1"], w["w2"], z, k, v, ws)
        grads = _grad_buffers(s, L)
        f32 = dict(dtype=torch.float32, device="cuda")
        scratch = dict(dk_part=torch.empty(s.S, s.h, **f32), dv_part=torch.empty(s.S, s.h, **f32),
                       dk=torch.empty(L, s.h, **f32), dv=torch.empty(L, s.h, **f32))
        TD.rank_backward(plan, rank, dz, x, g1, g2, k, v, ws, bws, grads, scratch)
        T.tsp_sync_status(plan)
        out = {n: t.float().cpu().numpy() for n, t in grads.items()}
        np.savez(os.path.join(out_dir, f"g{rank}.npz"), **out)
    finally:
        dist.destroy_process_group()


def test_two_processes_backward_against_oracle():
    import torch.multiprocessing as mp

    shape, seed = BWD_SHAPES[0]
    with tempfile.TemporaryDirectory() as out_dir:
        mp.start_processes(_rank_bwd_main, args=(shape.D, _free_port(), out_dir, vars(shape), seed),
                           nprocs=shape.D, join=True, start_method="spawn")
        gs = [dict(np.load(os.path.join(out_dir, f"g{r}.npz"))) for r in range(shape.D)]
    _, go = _oracle_grads(shape, make_layer_inputs(shape, seed))
    assert_close("dx", np.concatenate([g["dx"] for g in gs]).astype(np.float64), go["dx"])
    for n in GRADS:
        # every rank holds the same all-reduced sum
        assert np.array_equal(gs[0][n], gs[1][n]), n
        assert_close(n, gs[0][n].astype(np.float64), go[n])
