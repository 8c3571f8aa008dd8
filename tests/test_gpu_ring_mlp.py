"""The ring MLP on its own (tsp_ring_mlp_forward): with the layer's own
normalised activations b and fp32 residual stream y it reproduces the layer's
output bit for bit, and without a residual it matches the oracle's ring MLP
(tiny shape) element by element."""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import folded_tensor_sequence_map_b200 as T
import oracle as O
from synth_inputs import WORKLOADS, make_layer_inputs
from tests.gpu_helpers import GpuLayer, assert_close, host_f64, oracle_weights


@pytest.mark.parametrize("workload", ["tiny", "7b_s8k"])
def test_ring_mlp_reproduces_the_layer_mlp(workload):
    shape, seed = WORKLOADS[workload]
    inp = make_layer_inputs(shape, seed)
    layer = GpuLayer(shape, inp, training=True)
    S, h, D = shape.S, shape.h, shape.D
    z = layer.forward().clone()
    b = layer.saved_view("b", (S, h), torch.bfloat16).clone()
    y = layer.saved_view("y", (S, h), torch.float32).clone()
    ws = torch.empty(T.tsp_ring_mlp_workspace_size(layer.plan), dtype=torch.uint8, device="cuda")
    out = torch.full((S, h), float("nan"), dtype=torch.bfloat16, device="cuda")
    w = layer.w
    T.tsp_ring_mlp_forward(layer.plan, b, w["w1"], w["w2"], y, out, ws)
    T.tsp_sync_status(layer.plan)
    assert torch.equal(out, z)

    if workload == "tiny":
        zero = torch.zeros_like(y)
        T.tsp_ring_mlp_forward(layer.plan, b, w["w1"], w["w2"], zero, out, ws)
        T.tsp_sync_status(layer.plan)
        wo = oracle_weights(inp)
        ref = O.tsp_ring_mlp(host_f64(b), wo["w1"], wo["w2"], np.zeros((S, h)), D)
        assert_close("mid.mlp", host_f64(out), ref)
