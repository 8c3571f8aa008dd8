"""Shared pieces of the GPU parity tests: put seeded inputs on the device in
rank-major zigzag order, run the layer through the C ABI, bring results back,
and compare them with the oracle under the acceptance bounds."""

from __future__ import annotations

import json
import os
import time

import numpy as np
import torch

import folded_tensor_sequence_map_b200 as T
from synth_inputs import bits_to_f32
from tests.tolerances import bound_for

WEIGHTS = ("wqkv", "wo", "w1", "w2")


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


class GpuLayer:
    """Device buffers and one plan for a layer shape; forward/backward through the C ABI."""

    def __init__(self, shape, inp: dict, training: bool = True):
        self.shape = shape
        s = shape
        self.plan = T.tsp_plan(s.h, s.heads, s.ffn, s.S, s.D)
        self.zig = T.tsp_zigzag_map(self.plan)
        self.x = dev_bf16(inp["x"][self.zig])
        self.dy = dev_bf16(inp["dy"][self.zig]) if "dy" in inp else None
        self.w = {k: dev_bf16(inp[k]) for k in WEIGHTS}
        self.g1 = torch.from_numpy(inp["g1"]).cuda()
        self.g2 = torch.from_numpy(inp["g2"]).cuda()
        ws, saved = T.tsp_workspace_size(self.plan, training)
        self.ws = torch.empty(ws, dtype=torch.uint8, device="cuda")
        self.saved = torch.empty(saved, dtype=torch.uint8, device="cuda") if training else None
        self.y = torch.empty(s.S, s.h, dtype=torch.bfloat16, device="cuda")

    def forward(self):
        w = self.w
        T.tsp_layer_forward(self.plan, self.x, self.g1, w["wqkv"], w["wo"], self.g2, w["w1"], w["w2"], self.y,
                            self.saved, self.ws)
        T.tsp_sync_status(self.plan)
        return self.y

    def backward(self):
        s, w = self.shape, self.w
        dev = "cuda"
        self.grads = dict(
            dx=torch.empty(s.S, s.h, dtype=torch.bfloat16, device=dev),
            dg1=torch.empty(s.h, dtype=torch.float32, device=dev),
            dwqkv=torch.empty(3 * s.h, s.h, dtype=torch.float32, device=dev),
            dwo=torch.empty(s.h, s.h, dtype=torch.float32, device=dev),
            dg2=torch.empty(s.h, dtype=torch.float32, device=dev),
            dw1=torch.empty(s.ffn, s.h, dtype=torch.float32, device=dev),
            dw2=torch.empty(s.h, s.ffn, dtype=torch.float32, device=dev),
        )
        g = self.grads
        T.tsp_layer_backward(self.plan, self.dy, self.x, self.g1, w["wqkv"], w["wo"], self.g2, w["w1"], w["w2"],
                             self.saved, self.ws, g["dx"], g["dg1"], g["dwqkv"], g["dwo"], g["dg2"], g["dw1"],
                             g["dw2"])
        T.tsp_sync_status(self.plan)
        return g

    def saved_view(self, name: str, shape, dtype) -> torch.Tensor:
        off = T.tsp_test_buffer_offset(self.plan, name)
        buf = self.ws if name.startswith("ws.") else (self.saved if self.saved is not None else self.ws)
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        return buf[off:off + n].view(dtype).view(*shape)


def oracle_weights(inp: dict) -> dict:
    w = {k: bits_to_f32(inp[k]).astype(np.float64) for k in WEIGHTS}
    w["g1"] = inp["g1"].astype(np.float64)
    w["g2"] = inp["g2"].astype(np.float64)
    return w


def errors(gpu: np.ndarray, ref: np.ndarray):
    d = np.abs(gpu - ref)
    return float(d.max() / np.abs(ref).max()), float(d.mean() / np.abs(ref).mean())


def assert_close(name: str, gpu: np.ndarray, ref: np.ndarray, report: dict | None = None):
    assert gpu.shape == ref.shape, (name, gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{name}: non-finite values"
    mx, mn = errors(gpu, ref)
    bmax, bmean = bound_for(name)
    if report is not None:
        report[name] = (mx, mn)
    assert mx <= bmax and mn <= bmean, f"{name}: max-abs {mx:.3e} (bound {bmax:.1e}), mean-abs {mn:.3e} (bound {bmean:.1e})"


class OracleTimer:
    """Wall time of an oracle run inside a GPU test.  Printed always; appended
    as a JSON line to the file named by TSP_ORACLE_TIMES when that is set
    (how the oracle's host-side cost is measured on the GPU machine)."""

    def __init__(self, label: str, **meta):
        self.label, self.meta = label, meta

    def __enter__(self):
        self.t0 = time.perf_counter()
        return self

    def __exit__(self, *exc):
        sec = time.perf_counter() - self.t0
        rec = dict(label=self.label, seconds=round(sec, 2), cores=os.cpu_count(), **self.meta)
        print("oracle time", json.dumps(rec))
        path = os.environ.get("TSP_ORACLE_TIMES")
        if path and exc[0] is None:
            with open(path, "a") as f:
                f.write(json.dumps(rec) + "\n")
