"""One rank's share of the forward (``tsp_rank_forward_qkv`` / ``_out``), the
entry points for running the folded layer on D devices ("Zyphra TSP folds
TP+SP onto one GPU axis, 2.6x throughput on 1,024 MI300Xs", zubnet.ai,
paragraphs 1-2).

* On one device, the D ranks run in turn over shared K/V buffers (the
  all-gather then needs no copy): every rank's z rows, and the K/V they
  write, are bit for bit those of ``tsp_layer_forward`` (the same kernels on
  the same rows), for the tiny width with D = 2 and 4 and the 7B layer at
  S=4096, D=8.
* Two processes, one rank each, exchange K/V with torch.distributed (gloo,
  through host copies) as ``folded_tensor_sequence_map_b200.distributed``
  does on D GPUs; their z rows are again the layer's.  Both processes use the
  one GPU here; the kernels of one never wait on the other's.
"""

import os
import socket
import tempfile

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import folded_tensor_sequence_map_b200 as T
from synth_inputs import LayerShape, make_layer_inputs
from tests.gpu_helpers import GpuLayer, dev_bf16

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
