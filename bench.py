#!/usr/bin/env python
"""Benchmark of the folded TSP decoder layer on B200.

One step = one pass of the whole hot path: the layer forward (RMSNorm1, QKV
projection over the broadcast attention shards with the K/V all-gather in its
epilogue, causal attention over the zigzag layout, out-projection + residual,
RMSNorm2, W1 + GELU, ring-ordered W2 + residual) and its backward, over one
batch of seeded synthetic inputs (7B-shaped layer: h=4096, 32 heads x 128,
FFN 16384, S=131072 tokens, D=8 virtual ranks, bf16, weights N(0, 0.02),
x and dY N(0, 1), seed 4).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tsp|reference]

Prints one JSON line on rank 0.  With N > 1 (launched by torch.distributed.run)
every rank runs an independent replica of the same layer ("replicas only": the
folded layer's ranks are virtual ranks of one GPU), timed on the device and
reduced with MAX over ranks.  ``--impl reference`` times the fp64 CPU oracle on
the host cores instead (rank 0 only).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth_inputs import WORKLOADS, LayerShape, make_layer_inputs  # noqa: E402

METRIC = "TSP layer tokens/s (fwd, fwd+bwd) at S=128K, D=8; % bf16 tensor-core peak"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "7b_s128k"
# oracle samples: the same 7B layer (fwd+bwd) at these token counts; the
# reference arm times the first, cpu_baseline times both
CPU_SAMPLE_S = (1024, 2048)
NOMINAL_TFLOPS = 2250.0   # dense bf16/fp16 datasheet figure
NOMINAL_MHZ = 1965.0      # clocks.max.sm of this part

# DRAM bytes (read + write) of one launch from an ncu capture of the current
# kernel build (dram__bytes_read.sum + dram__bytes_write.sum, one ncu pass, at
# the benchmark's size), and the S of that capture.  At another S the figure
# is scaled by S, which holds only while re-reads stay in L2.  Must be
# re-measured (or removed) whenever the kernel changes.
MEASURED_TRAFFIC = {"bwd_attn_fused": (138.10e9 + 94.23e9, 131072)}


def peaks():
    """(burst TFLOP/s, sustained TFLOP/s, HBM GB/s, source): the measured copy
    bandwidth and cuBLAS GEMM rates of this machine's B200s when the driver has
    written them, else an earlier measurement on this machine (fp16 and bf16
    dense MMAs have the same rate)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p["bf16_tflops"], p["bf16_tflops_sustained"], p["hbm_gbs"], "measured"
    except (OSError, KeyError, ValueError):
        return 1590.0, 1400.0, 6650.0, "fallback (earlier measurement on this pool)"


def layer_flops(s: LayerShape, backward: bool) -> float:
    """Algorithmic FLOPs of the forward (backward=False) or of the backward
    alone (backward=True, twice the forward); a step is their sum."""
    fwd = 2.0 * s.S * (4.0 * s.h * s.h + 2.0 * s.h * s.ffn) + 2.0 * s.h * s.S * (s.S + 1.0)
    return 2.0 * fwd if backward else fwd


def step_flops(s: LayerShape) -> float:
    return layer_flops(s, False) + layer_flops(s, True)


def stage_flops(s: LayerShape) -> dict:
    """Algorithmic FLOPs of one launch of each stage (causal pairs only, no recompute)."""
    S, h, F = float(s.S), float(s.h), float(s.ffn)
    att = h * S * (S + 1.0)
    return {
        "fwd_qkv_gemm": 6 * S * h * h, "fwd_attention": 2 * att, "fwd_out_proj_gemm": 2 * S * h * h,
        "fwd_w1_gelu_gemm": 2 * S * h * F, "fwd_w2_ring_gemm": 2 * S * h * F,
        "bwd_dgelu_gemm": 2 * S * h * F, "bwd_dw2_gemm": 2 * S * h * F, "bwd_dw1_gemm": 2 * S * h * F,
        "bwd_db_ring_gemm": 2 * S * h * F, "bwd_do_gemm": 2 * S * h * h, "bwd_dwo_gemm": 2 * S * h * h,
        "bwd_attn_dkdv": 3 * att, "bwd_attn_dq": att, "bwd_dwqkv_gemm": 6 * S * h * h, "bwd_da_gemm": 6 * S * h * h,
        "bwd_attn_fused": 4 * att,
    }


def inactive_stages(s: LayerShape) -> set:
    """Stages that the layer does not run for this shape: head size 128
    takes the single-pass attention backward, other head sizes the two
    kernels; the dK/dV conversion belongs to the per-rank backward only."""
    attn = {"bwd_attn_dkdv", "bwd_attn_dq"} if s.dh == 128 else {"bwd_attn_fused", "bwd_attn_dq_convert"}
    return attn | {"bwd_convert_dkdv"}


def hbm_stage_bytes(s: LayerShape) -> dict:
    """Algorithmic HBM bytes of one launch of each memory-bound stage: every
    tensor the stage reads or writes, once (gains and norm statistics
    included; the dg partial sums are written and read back once)."""
    S, h, H = float(s.S), float(s.h), float(s.heads)
    partials = S / 64 * h * 4
    wts = (4.0 * h * h + 2.0 * h * s.ffn) * 2                             # the four weights, 16-bit
    return {
        "fwd_convert_weights": 3 * wts,                                   # read twice (max, convert), write fp16
        "fwd_rmsnorm1": S * h * (2 + 2) + S * 4 + h * 4,                  # x bf16 -> a fp16, rstd
        "fwd_rmsnorm2": S * h * (4 + 2) + S * 4 + h * 4,                  # y f32 -> b fp16, rstd
        "bwd_convert_dy": 3 * S * h * 2,                                  # dY read twice, fp16 copy written
        "bwd_rmsnorm2": S * h * (4 + 4 + 2 + 4 + 2) + S * 4 + 2 * partials + h * 8,  # db, y, dY -> dy f32+fp16
        "bwd_rmsnorm1": S * h * (4 + 2 + 4 + 2) + S * 4 + 2 * partials + h * 8,      # da, x, dy -> dx bf16
        # O, dO -> delta f32 [H][S]; head size 128 also reads K, V for the dQ
        # bound and clears the 32-bit dQ sum
        "bwd_attn_delta": S * h * (2 + 2) + S * H * 4 + (S * h * (2 + 2 + 4) if s.dh == 128 else 0),
        "bwd_attn_dq_convert": S * h * (4 + 2),                           # dQ sum f32 -> dQ fp16
        "bwd_convert_dkdv": 2 * S / s.D * h * (4 + 2),                    # one rank's dK, dV f32 -> fp16
    }


# ---------------------------------------------------------------------------
# multi-process plumbing (N > 1: independent replicas)
# ---------------------------------------------------------------------------

def dist_setup(backend: str):
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1 and not dist.is_initialized():
        import datetime

        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))
    return int(os.environ.get("RANK", "0")), world


def reduce_max(value: float, device=None) -> float:
    """MAX of a per-rank float over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, flag in zip(self.NAMES, parts[3:7]):
                if flag.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and --impl reference)
# ---------------------------------------------------------------------------

def oracle_sample_seconds(shape: LayerShape, seed: int, S: int) -> float:
    """Wall time of the fp64 oracle's folded forward + backward of the same
    layer at S tokens (inputs drawn and converted outside the timed part)."""
    import oracle as O
    from synth_inputs import bits_to_f32

    s = LayerShape(h=shape.h, heads=shape.heads, ffn=shape.ffn, S=S, D=shape.D)
    inp = make_layer_inputs(s, seed)
    zig = O.zigzag_map(s.S, s.D).ravel()
    w = {k: bits_to_f32(inp[k]).astype(np.float64) for k in ("wqkv", "wo", "w1", "w2")}
    w["g1"] = inp["g1"].astype(np.float64)
    w["g2"] = inp["g2"].astype(np.float64)
    x = bits_to_f32(inp["x"][zig]).astype(np.float64)
    dy = bits_to_f32(inp["dy"][zig]).astype(np.float64)
    t0 = time.perf_counter()
    _, cache = O.tsp_layer_forward(x, w, s.heads, s.D)
    O.tsp_layer_backward(dy, w, cache)
    return time.perf_counter() - t0


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:  # noqa: BLE001
        pass
    return os.cpu_count() or 1


def project_two_sizes(t1: float, s1: int, t2: float, s2: int, S: int) -> float:
    """Seconds at S from a fit T(s) = a s + b s^2 through two measured runs:
    the token-local work grows with s, the causal attention with s^2."""
    b = (t2 / s2 - t1 / s1) / (s2 - s1)
    a = t1 / s1 - b * s1
    return max(a, 0.0) * S + max(b, 0.0) * S * S


def cpu_baseline(shape: LayerShape, seed: int) -> dict:
    """The oracle timed on this host at the two sample sizes.  `value` is what
    was timed: tokens/s of the larger sample; the S=131072 figure is a
    projection, in its own field."""
    (s1, s2) = CPU_SAMPLE_S
    t1 = oracle_sample_seconds(shape, seed, s1)
    t2 = oracle_sample_seconds(shape, seed, s2)
    proj = project_two_sizes(t1, s1, t2, s2, shape.S)
    return {
        "value": s2 / t2,
        "unit": UNIT,
        "cores": cpu_threads(),
        "kind": "oracle",
        "sample": (f"fp64 NumPy oracle, folded forward+backward of the same 7B layer (D={shape.D}) at "
                   f"S={s2}: {t2:.2f} s measured, one run (value = {s2} tokens / {t2:.2f} s); also S={s1}: "
                   f"{t1:.2f} s measured"),
        "projected_to_S": shape.S,
        "projected_value": shape.S / proj,
        "projection": f"T(S) = a S + b S^2 through the two measured runs: {proj:.0f} s at S={shape.S}",
    }


def run_reference(args, shape: LayerShape, seed: int):
    """--impl reference: the oracle itself, timed on the host cores.  One step
    is the oracle's folded forward + backward of the same layer at the first
    sample size; `value` and `ms_per_step` describe exactly the timed steps."""
    rank, world = int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    S = CPU_SAMPLE_S[0]
    for _ in range(args.warmup):
        oracle_sample_seconds(shape, seed, S)
    secs = [oracle_sample_seconds(shape, seed, S) for _ in range(args.steps)]
    total = sum(secs)
    value = S * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "h": shape.h, "heads": shape.heads, "ffn": shape.ffn, "seq_len": shape.S,
                   "D": shape.D, "global_batch": 1, "parallelism": "virtual ranks on one device",
                   "l2": "inputs larger than L2", "timed_sample_seq_len": S},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                         "sample": (f"fp64 NumPy oracle, folded forward+backward of the same 7B layer at S={S}, "
                                    f"D={shape.D}: {args.steps} timed runs, {total:.2f} s in all "
                                    f"(median {statistics.median(secs):.2f} s); value = tokens timed / seconds")},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU run: a stack of layers (--layers)
# ---------------------------------------------------------------------------

def run_stack(args, shape: LayerShape, seed: int):
    """One step = forward + backward of `layers` folded layers with
    activation recompute (tsp_stack_forward / tsp_stack_backward).  For
    timing, every layer holds its own device copy of one layer's drawn
    weights (the values do not change the work).  Algorithmic FLOPs count
    each layer's forward and backward once; the recomputed forwards are
    reported apart."""
    import torch

    import folded_tensor_sequence_map_b200 as T

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    rank, world = dist_setup("nccl")
    n, S, h, F = args.layers, shape.S, shape.h, shape.ffn
    bf = torch.bfloat16
    plan = T.tsp_plan(shape.h, shape.heads, shape.ffn, shape.S, shape.D)
    zig = T.tsp_zigzag_map(plan)
    inp = make_layer_inputs(shape, seed)
    to_dev = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(bf).to(dev)
    x = torch.from_numpy(np.ascontiguousarray(inp["x"][zig]).view(np.int16)).view(bf).to(dev)
    dz = torch.from_numpy(np.ascontiguousarray(inp["dy"][zig]).view(np.int16)).view(bf).to(dev)
    W = {k: [to_dev(inp[k]) for _ in range(n)] for k in ("wqkv", "wo", "w1", "w2")}
    G = {k: [torch.from_numpy(inp[k]).to(dev) for _ in range(n)] for k in ("g1", "g2")}
    del inp
    ws_n, saved_n, inputs_n = T.tsp_stack_workspace_size(plan, n)
    ws = torch.empty(ws_n, dtype=torch.uint8, device=dev)
    saved = torch.empty(saved_n, dtype=torch.uint8, device=dev)
    inputs = torch.empty(inputs_n, dtype=torch.uint8, device=dev)
    z = torch.empty(S, h, dtype=bf, device=dev)
    dx = torch.empty(S, h, dtype=bf, device=dev)
    grads = {"dg1": [torch.empty(h, device=dev) for _ in range(n)],
             "dwqkv": [torch.empty(3 * h, h, device=dev) for _ in range(n)],
             "dwo": [torch.empty(h, h, device=dev) for _ in range(n)],
             "dg2": [torch.empty(h, device=dev) for _ in range(n)],
             "dw1": [torch.empty(F, h, device=dev) for _ in range(n)],
             "dw2": [torch.empty(h, F, device=dev) for _ in range(n)]}
    stream = torch.cuda.current_stream(dev)
    wargs = (G["g1"], W["wqkv"], W["wo"], G["g2"], W["w1"], W["w2"])

    def step():
        T.tsp_stack_forward(plan, x, *wargs, z, inputs, saved, ws, stream)
        T.tsp_stack_backward(plan, dz, x, *wargs, inputs, saved, ws, dx, grads["dg1"], grads["dwqkv"],
                             grads["dwo"], grads["dg2"], grads["dw1"], grads["dw2"], stream)

    for _ in range(args.warmup):
        step()
    T.tsp_sync_status(plan, stream)
    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local)
    launches0 = T.tsp_kernel_launches(plan)
    with ClockSampler(gpu_id) as clk:
        barrier(dev)
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            step()
        b.record(stream)
        torch.cuda.synchronize(dev)
        barrier(dev)
    T.tsp_sync_status(plan, stream)
    t = reduce_max(a.elapsed_time(b) / 1e3, dev)
    launches = T.tsp_kernel_launches(plan) - launches0
    burst, sustained, _, src = peaks()
    flops = n * step_flops(shape)
    recompute = (n - 1) * layer_flops(shape, False)
    line = {
        "metric": f"TSP stack tokens/s (fwd+bwd, {n} layers, activation recompute) at S={S}, D={shape.D}",
        "value": world * S * args.steps / t, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic (every layer a copy of one layer's drawn weights)",
        "config": {"workload": f"{args.workload}_stack{n}" + (f"_seq{S}" if args.seq else ""), "layers": n, "h": h, "heads": shape.heads, "ffn": F,
                   "seq_len": S, "D": shape.D, "global_batch": 1,
                   "parallelism": "virtual ranks on one device; replicas across GPUs",
                   "l2": "inputs larger than L2"},
        "fwd_bwd_frac_of_bf16_peak": flops * args.steps / t / 1e12 / sustained,
        "with_recompute_frac_of_bf16_peak": (flops + recompute) * args.steps / t / 1e12 / sustained,
        "peak_source": f"{src} sustained {sustained} TFLOP/s",
        "device_memory_gb": round(torch.cuda.max_memory_allocated(dev) / 1e9, 1),
        "gpu_launches": int(launches),
        "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# GPU run
# ---------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="tsp", choices=["tsp", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu", action="store_true", help="skip the cpu_baseline leg")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg")
    ap.add_argument("--seq", type=int, default=0, help="override S of the workload (profiling runs)")
    ap.add_argument("--ranks", type=int, default=0, help="override D of the workload (D sweep)")
    ap.add_argument("--layers", type=int, default=1,
                    help="time a stack of this many layers with activation recompute instead of one layer")
    args = ap.parse_args()
    shape, seed = WORKLOADS[args.workload]
    if args.seq or args.ranks:
        shape = LayerShape(h=shape.h, heads=shape.heads, ffn=shape.ffn, S=args.seq or shape.S,
                           D=args.ranks or shape.D)
    if args.impl == "reference":
        run_reference(args, shape, seed)
        return
    if args.layers > 1:
        run_stack(args, shape, seed)
        return

    import torch

    import folded_tensor_sequence_map_b200 as T

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    rank, world = dist_setup("nccl")
    bf = torch.bfloat16

    plan = T.tsp_plan(shape.h, shape.heads, shape.ffn, shape.S, shape.D)
    zig = T.tsp_zigzag_map(plan)
    inp = make_layer_inputs(shape, seed)
    to_dev = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(bf).to(dev)
    x_host = torch.from_numpy(np.ascontiguousarray(inp["x"][zig]).view(np.int16)).view(bf).pin_memory()
    dy_host = torch.from_numpy(np.ascontiguousarray(inp["dy"][zig]).view(np.int16)).view(bf).pin_memory()
    W = {k: to_dev(inp[k]) for k in ("wqkv", "wo", "w1", "w2")}
    g1 = torch.from_numpy(inp["g1"]).to(dev)
    g2 = torch.from_numpy(inp["g2"]).to(dev)
    del inp
    x = x_host.to(dev)
    dy = dy_host.to(dev)
    S, h, F = shape.S, shape.h, shape.ffn
    ws_n, saved_n = T.tsp_workspace_size(plan, True)
    ws = torch.empty(ws_n, dtype=torch.uint8, device=dev)
    saved = torch.empty(saved_n, dtype=torch.uint8, device=dev)
    y = torch.empty(S, h, dtype=bf, device=dev)
    grads = dict(dx=torch.empty(S, h, dtype=bf, device=dev), dg1=torch.empty(h, device=dev),
                 dwqkv=torch.empty(3 * h, h, device=dev), dwo=torch.empty(h, h, device=dev),
                 dg2=torch.empty(h, device=dev), dw1=torch.empty(F, h, device=dev), dw2=torch.empty(h, F, device=dev))
    stream = torch.cuda.current_stream(dev)

    def fwd():
        T.tsp_layer_forward(plan, x, g1, W["wqkv"], W["wo"], g2, W["w1"], W["w2"], y, saved, ws, stream)

    def bwd():
        g = grads
        T.tsp_layer_backward(plan, dy, x, g1, W["wqkv"], W["wo"], g2, W["w1"], W["w2"], saved, ws, g["dx"],
                             g["dg1"], g["dwqkv"], g["dwo"], g["dg2"], g["dw1"], g["dw2"], stream)

    def timed(fn, steps):
        barrier(dev)
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        barrier(dev)
        T.tsp_sync_status(plan, stream)
        return reduce_max(a.elapsed_time(b) / 1e3, dev)

    step = lambda: (fwd(), bwd())
    for _ in range(args.warmup):
        step()
    T.tsp_sync_status(plan, stream)

    # fwd+bwd: the headline, with per-stage events and clocks
    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local)
    launches0 = T.tsp_kernel_launches(plan)
    T.tsp_profile_enable(plan, True)
    with ClockSampler(gpu_id) as clk:
        t_step = timed(step, args.steps)
    launches = T.tsp_kernel_launches(plan) - launches0
    stages = {}
    for i in range(T.TSP_NUM_STAGES):
        name, ms, calls, nk = T.tsp_profile_read(plan, i)
        stages[name] = (ms, calls, nk)
    T.tsp_profile_enable(plan, False)
    for _ in range(2):
        fwd()
    t_fwd = timed(fwd, args.steps)

    # end to end: pinned host inputs in, results out, inside the timed region.
    # Every step copies its own inputs in and its results out; the copies run
    # on two copy streams beside the compute (inputs and outputs double-
    # buffered: step i+1's inputs arrive and step i's results leave while
    # step i / i+1 computes), and the timed region runs from before the first
    # step's input copy to after the last step's result copy.
    e2e = None
    if not args.no_e2e:
        y_host = torch.empty(S, h, dtype=bf).pin_memory()
        g_host = {k: torch.empty_like(v, device="cpu").pin_memory() for k, v in grads.items()}
        ins = [(x, dy), (torch.empty_like(x), torch.empty_like(dy))]
        outs = [(y, grads), (torch.empty_like(y), {k: torch.empty_like(v) for k, v in grads.items()})]
        h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: [torch.cuda.Event(), torch.cuda.Event()]
        x_ready, dy_ready, in_free, z_ready, out_ready, out_free = ev(), ev(), ev(), ev(), ev(), ev()

        def copy_in(b):
            # x first: the forward needs only x, dY is read from the backward on
            with torch.cuda.stream(h2d):
                ins[b][0].copy_(x_host, non_blocking=True)
                x_ready[b].record(h2d)
                ins[b][1].copy_(dy_host, non_blocking=True)
                dy_ready[b].record(h2d)

        def e2e_run(steps):
            start = torch.cuda.Event()
            start.record(stream)
            h2d.wait_event(start)
            d2h.wait_event(start)
            copy_in(0)
            for i in range(steps):
                b, nb = i % 2, (i + 1) % 2
                if i + 1 < steps:
                    if i >= 1:
                        h2d.wait_event(in_free[nb])     # step i-1 has finished reading them
                    copy_in(nb)
                stream.wait_event(x_ready[b])
                if i >= 2:
                    stream.wait_event(out_free[b])      # step i-2's results have left
                xi, dyi = ins[b]
                yo, go = outs[b]
                T.tsp_layer_forward(plan, xi, g1, W["wqkv"], W["wo"], g2, W["w1"], W["w2"], yo, saved, ws, stream)
                z_ready[b].record(stream)
                stream.wait_event(dy_ready[b])
                T.tsp_layer_backward(plan, dyi, xi, g1, W["wqkv"], W["wo"], g2, W["w1"], W["w2"], saved, ws,
                                     go["dx"], go["dg1"], go["dwqkv"], go["dwo"], go["dg2"], go["dw1"], go["dw2"],
                                     stream)
                in_free[b].record(stream)
                out_ready[b].record(stream)
                # z leaves while the backward runs, the gradients after it
                d2h.wait_event(z_ready[b])
                with torch.cuda.stream(d2h):
                    y_host.copy_(yo, non_blocking=True)
                d2h.wait_event(out_ready[b])
                with torch.cuda.stream(d2h):
                    for k, v in go.items():
                        g_host[k].copy_(v, non_blocking=True)
                out_free[b].record(d2h)
            stream.wait_stream(h2d)
            stream.wait_stream(d2h)

        e2e_run(2)
        barrier(dev)
        torch.cuda.synchronize(dev)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e2e_run(args.steps)
        b_.record(stream)
        torch.cuda.synchronize(dev)
        barrier(dev)
        T.tsp_sync_status(plan, stream)
        t_e2e = reduce_max(a.elapsed_time(b_) / 1e3, dev)
        d2h_bytes = y.numel() * y.element_size() + sum(v.numel() * v.element_size() for v in grads.values())
        e2e = {"value": world * S * args.steps / t_e2e, "unit": UNIT,
               "h2d_bytes_per_step": x.numel() * 2 + dy.numel() * 2, "d2h_bytes_per_step": d2h_bytes,
               "copied": "x, dY in; z, dx, dg1, dWqkv, dWo, dg2, dW1, dW2 out (pinned host memory), every step; "
                         "on two copy streams overlapping the compute (inputs and outputs double-buffered; "
                         "dY arrives during the forward, z leaves during the backward), "
                         "timed from before the first input copy to after the last result copy"}

    burst, sustained, hbm, src = peaks()
    flops = stage_flops(shape)
    total_ms = sum(v[0] for v in stages.values())
    dom = max((k for k in flops), key=lambda k: stages[k][0])
    dom_ms = stages[dom][0] / max(stages[dom][1], 1)
    achieved = flops[dom] / (dom_ms / 1e3) / 1e12
    value = world * S * args.steps / t_step
    fwd_value = world * S * args.steps / t_fwd
    frac_step = step_flops(shape) * args.steps / t_step / 1e12 / sustained
    frac_fwd = layer_flops(shape, False) * args.steps / t_fwd / 1e12 / sustained
    clocks = clk.summary()
    run_mhz = clocks.get("sm_mhz") or NOMINAL_MHZ
    # the datasheet dense peak taken at the run's median SM clock: the tensor
    # pipe's rate scales with the clock, and the power cap sets the clock
    at_clock = NOMINAL_TFLOPS * run_mhz / NOMINAL_MHZ
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t_step / args.steps * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16", "data": "synthetic",
        "dtype_note": ("bf16 inputs and outputs; every tensor-core operand is fp16 (exact power-of-two-scaled "
                       "copies of the bf16 weights and dY, fp16 intermediates), fp32 accumulation; fp16 and "
                       "bf16 dense MMAs have the same rate"),
        "config": {"workload": args.workload, "h": h, "heads": shape.heads, "ffn": F, "seq_len": S, "D": shape.D,
                   "global_batch": 1, "parallelism": "virtual ranks on one device; replicas across GPUs",
                   "l2": "inputs larger than L2 (1 GiB activations per tensor)"},
        "fwd": {"value": fwd_value, "unit": UNIT, "ms": t_fwd / args.steps * 1e3,
                "frac_of_bf16_peak": frac_fwd},
        "fwd_bwd_frac_of_bf16_peak": frac_step,
        "fwd_bwd_frac_of_bf16_burst_peak": frac_step * sustained / burst,
        "fwd_bwd_frac_of_nominal_at_run_clock": frac_step * sustained / at_clock,
        "fwd_frac_of_bf16_burst_peak": frac_fwd * sustained / burst,
        "fwd_frac_of_nominal_at_run_clock": frac_fwd * sustained / at_clock,
        "peak_source": (f"{src} (sustained {sustained} TFLOP/s for the step fractions, burst {burst}; "
                        f"nominal {NOMINAL_TFLOPS:.0f} TFLOP/s at {NOMINAL_MHZ:.0f} MHz scaled to the run's "
                        f"median {run_mhz:.0f} MHz = {at_clock:.0f} TFLOP/s)"),
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": sustained, "unit": "TFLOP/s",
                     "frac": achieved / sustained, "frac_of_burst": achieved / burst,
                     "frac_of_nominal_at_run_clock": achieved / at_clock,
                     "traffic": (MEASURED_TRAFFIC[dom][0] * S / MEASURED_TRAFFIC[dom][1]) if dom in MEASURED_TRAFFIC
                     else None,
                     "traffic_note": ("not measured for this kernel build" if dom not in MEASURED_TRAFFIC
                                      else "ncu dram bytes of one launch at this S" if MEASURED_TRAFFIC[dom][1] == S
                                      else "ncu dram bytes of one launch at another S scaled by S"),
                     "peak_note": f"{src} sustained bf16 (kernel timed inside a long step)"},
        "hbm_stages": {k: {"bytes": b, "ms": stages[k][0] / max(stages[k][1], 1),
                           "achieved": b / (stages[k][0] / max(stages[k][1], 1) / 1e3) / 1e9,
                           "peak": hbm, "unit": "GB/s",
                           "frac": b / (stages[k][0] / max(stages[k][1], 1) / 1e3) / 1e9 / hbm}
                       for k, b in hbm_stage_bytes(shape).items() if stages.get(k, (0, 0))[0] > 0},
        "hbm_peak_note": f"{src} HBM copy bandwidth",
        "stage_ms_per_step": {k: round(v[0] / max(v[1], 1), 4) for k, v in stages.items()},
        "stage_share": {k: round(v[0] / total_ms, 4) for k, v in stages.items()},
        "gpu_launches": int(launches),
        "clocks": clocks,
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(shape, seed)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del plan
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
