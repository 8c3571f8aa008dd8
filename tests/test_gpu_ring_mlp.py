"""The ring MLP on its own (tsp_ring_mlp_forward) against the oracle's ring
MLP, element by element under the stated bounds: with the layer's own
normalised activations b (rounded to the entry point's bf16 input) and fp32
residual stream y, and (tiny shape) without a residual."""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import folded_tensor_sequence_map_b200 as T
import oracle as O
from synth_inputs import WORKLOADS, make_layer_inputs
from tests.gpu_helpers import GpuLayer, assert_close, host_f64, oracle_weights


@pytest.mark.parametrize("workload", ["tiny", "7b_s8k"])
def test_ring_mlp_matches_the_oracle(workload):
    shape, seed = WORKLOADS[workload]
    inp = make_layer_inputs(shape, seed, with_dy=False)
    layer = GpuLayer(shape, inp, training=True)
    S, h, D = shape.S, shape.h, shape.D
    layer.forward()
    b = layer.saved_view("b", (S, h), torch.float16).to(torch.bfloat16).contiguous()
    y = layer.saved_view("y", (S, h), torch.float32).clone()
    ws = torch.empty(T.tsp_ring_mlp_workspace_size(layer.plan), dtype=torch.uint8, device="cuda")
    out = torch.full((S, h), float("nan"), dtype=torch.bfloat16, device="cuda")
    w = layer.w
    wo = oracle_weights(inp)
    T.tsp_ring_mlp_forward(layer.plan, b, w["w1"], w["w2"], y, out, ws)
    T.tsp_sync_status(layer.plan)
    ref = O.tsp_ring_mlp(host_f64(b), wo["w1"], wo["w2"], host_f64(y), D)
    assert_close("mlp", host_f64(out), ref)

    if workload == "tiny":
        zero = torch.zeros_like(y)
        T.tsp_ring_mlp_forward(layer.plan, b, w["w1"], w["w2"], zero, out, ws)
        T.tsp_sync_status(layer.plan)
        ref = O.tsp_ring_mlp(host_f64(b), wo["w1"], wo["w2"], np.zeros((S, h)), D)
        assert_close("mlp", host_f64(out), ref)


def test_fp16_overflow_is_reported():
    # b is copied to fp16 unscaled; a magnitude fp16 cannot hold must come back
    # as TSP_ERR_RANGE from tsp_sync_status, and the flag is cleared by that report
    shape, seed = WORKLOADS["tiny"]
    inp = make_layer_inputs(shape, seed, with_dy=False)
    S, h = shape.S, shape.h
    plan = T.tsp_plan(shape.h, shape.heads, shape.ffn, S, shape.D)
    from tests.gpu_helpers import dev_bf16

    w1, w2 = dev_bf16(inp["w1"]), dev_bf16(inp["w2"])
    b = torch.randn(S, h, device="cuda").to(torch.bfloat16)
    b[3, 5] = 1.0e5
    resid = torch.zeros(S, h, dtype=torch.float32, device="cuda")
    out = torch.empty(S, h, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(T.tsp_ring_mlp_workspace_size(plan), dtype=torch.uint8, device="cuda")
    T.tsp_ring_mlp_forward(plan, b, w1, w2, resid, out, ws)
    with pytest.raises(T.TSPError) as e:
        T.tsp_sync_status(plan)
    assert T.STATUS_NAMES[e.value.status] == "TSP_ERR_RANGE"
    T.tsp_sync_status(plan)
