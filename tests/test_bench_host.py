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
        f = bench.stage_flops(s)
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
