"""Host logic of bench.py without a GPU: the max-over-ranks reduction with two
gloo ranks on CPU, the FLOP bookkeeping, and the clock-log parser."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from synth_inputs import WORKLOADS


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    r, w = bench.dist_setup("gloo")
    assert (r, w) == (rank, world)
    bench.barrier()
    out[rank] = bench.reduce_max(1.5 + rank)
    dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    assert dict(out) == {0: 2.5, 1: 2.5}


def test_single_process_reduce_is_identity():
    assert bench.reduce_max(3.25) == 3.25


def test_stage_flops_sum_to_layer_flops():
    for name in ("tiny", "7b_s8k", "7b_s128k"):
        s, _ = WORKLOADS[name]
        skip = bench.inactive_stages(s)
        f = {k: v for k, v in bench.stage_flops(s).items() if k not in skip}
        fwd = sum(v for k, v in f.items() if k.startswith("fwd_"))
        bwd = sum(v for k, v in f.items() if k.startswith("bwd_"))
        assert fwd == pytest.approx(bench.layer_flops(s, False), rel=1e-12)
        assert bwd == pytest.approx(bench.layer_flops(s, True), rel=1e-12)


def test_clock_summary_parses_reasons():
    c = bench.ClockSampler("0")
    c.lines = ["1800, 1965, 900.5, Not Active, Not Active, Not Active, Active",
               "1900, 1965, 950.0, Not Active, Not Active, Not Active, Not Active",
               "garbage"]
    s = c.summary()
    assert s["sm_mhz"] == 1850 and s["sm_max_mhz"] == 1965 and s["reasons"] == ["sw_power_cap"]


def test_stage_accounting_covers_every_library_stage_once():
    """Each library stage is either a contraction (FLOPs) or memory-bound
    (bytes), never both and never neither."""
    import folded_tensor_sequence_map_b200 as T

    s, _ = WORKLOADS["7b_s128k"]
    p = T.tsp_plan(s.h, s.heads, s.ffn, s.S, s.D)
    names = {T.tsp_profile_read(p, i)[0] for i in range(T.TSP_NUM_STAGES)}
    flops, hbm = set(bench.stage_flops(s)), set(bench.hbm_stage_bytes(s))
    assert not flops & hbm
    assert flops | hbm == names


def test_hbm_stage_bytes_of_the_forward_norm():
    """RMSNorm1 forward at the 7B shape reads x and writes a (bf16, 1 GiB
    each) plus rstd and the gain."""
    s, _ = WORKLOADS["7b_s128k"]
    b = bench.hbm_stage_bytes(s)
    assert b["fwd_rmsnorm1"] == 2 * 2 * s.S * s.h + 4 * s.S + 4 * s.h
    assert all(v > 0 for v in b.values())
