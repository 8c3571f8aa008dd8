"""Inference prefill (tsp_layer_prefill): the forward without training state,
leaving the layer's keys and values in caller-owned caches in global position
order.  Checked bit for bit against the training forward's own output and
K/V, and (tiny shape) against the oracle's gathered K/V and output."""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import folded_tensor_sequence_map_b200 as T
import oracle as O
from synth_inputs import WORKLOADS, bits_to_f32, make_layer_inputs
from tests.gpu_helpers import GpuLayer, assert_close, host_f64, oracle_weights


@pytest.mark.parametrize("workload", ["tiny", "7b_s8k"])
def test_prefill_matches_forward_and_fills_caches(workload):
    shape, seed = WORKLOADS[workload]
    inp = make_layer_inputs(shape, seed)
    layer = GpuLayer(shape, inp, training=True)
    S, h = shape.S, shape.h
    y_fwd = layer.forward().clone()
    k_fwd = layer.saved_view("k", (S, h), torch.float16).clone()
    v_fwd = layer.saved_view("v", (S, h), torch.float16).clone()

    ws_n, saved_n = T.tsp_workspace_size(layer.plan, False)
    assert saved_n == 0
    ws = torch.empty(ws_n, dtype=torch.uint8, device="cuda")
    y = torch.full((S, h), float("nan"), dtype=torch.bfloat16, device="cuda")
    kc = torch.full((S, h), float("nan"), dtype=torch.float16, device="cuda")
    vc = torch.full((S, h), float("nan"), dtype=torch.float16, device="cuda")
    w = layer.w
    T.tsp_layer_prefill(layer.plan, layer.x, layer.g1, w["wqkv"], w["wo"], layer.g2, w["w1"], w["w2"], y, kc, vc, ws)
    T.tsp_sync_status(layer.plan)

    assert torch.equal(y, y_fwd)
    assert torch.equal(kc, k_fwd)
    assert torch.equal(vc, v_fwd)
    if workload == "tiny":
        xl = bits_to_f32(inp["x"][layer.zig]).astype(np.float64)
        zo, cache = O.tsp_layer_forward(xl, oracle_weights(inp), shape.heads, shape.D)
        assert_close("mid.k", host_f64(kc), cache["Kg"])
        assert_close("mid.v", host_f64(vc), cache["Vg"])
        assert_close("z", host_f64(y), zo)
