"""A stack of folded layers with activation recompute (``tsp_stack_*``)
against the oracle's stack, and against the layer entry points.

The model the pages measure is a stack of 32 such layers ("Zyphra TSP folds
TP+SP onto one GPU axis, 2.6x throughput on 1,024 MI300Xs", zubnet.ai,
paragraph 1).  Checked here:
* tiny shape, 3 layers, and the 7B layer at S=4096, D=8, 2 layers: z, dx and
  every layer's six parameter gradients against
  ``oracle.tsp_stack_forward/backward`` (bf16 tensors between layers) within
  the stack's bound: the stated mean bound times sqrt(layers), one more bf16
  rounding per layer on every tensor's path (tests/tolerances.py);
* the stack's results are bit for bit those of calling the layer entry points
  by hand (forward of every layer with its own saved buffer, then backward
  from the top), so the recompute changes nothing;
* the inference forward (saved = NULL) gives the same z bit for bit.
"""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import folded_tensor_sequence_map_b200 as T
import oracle as O
from synth_inputs import LayerShape, bits_to_f32, make_stack_inputs
from tests.gpu_helpers import OracleTimer, dev_bf16, errors, host_f64, oracle_weights
from tests.tolerances import stack_bound_for

GRADS = ("dg1", "dwqkv", "dwo", "dg2", "dw1", "dw2")


class GpuStack:
    def __init__(self, shape, layers, seed):
        s = shape
        self.shape, self.n = s, layers
        self.inp = make_stack_inputs(s, layers, seed)
        self.plan = T.tsp_plan(s.h, s.heads, s.ffn, s.S, s.D)
        self.zig = T.tsp_zigzag_map(self.plan)
        self.x = dev_bf16(self.inp["x"][self.zig])
        self.dz = dev_bf16(self.inp["dy"][self.zig])
        L = self.inp["layers"]
        self.w = {k: [dev_bf16(lw[k]) for lw in L] for k in ("wqkv", "wo", "w1", "w2")}
        self.g = {k: [torch.from_numpy(lw[k]).cuda() for lw in L] for k in ("g1", "g2")}
        ws, saved, inputs = T.tsp_stack_workspace_size(self.plan, layers)
        self.ws = torch.empty(ws, dtype=torch.uint8, device="cuda")
        self.saved = torch.empty(saved, dtype=torch.uint8, device="cuda")
        self.inputs = torch.empty(max(inputs, 16), dtype=torch.uint8, device="cuda")
        self.z = torch.empty(s.S, s.h, dtype=torch.bfloat16, device="cuda")

    def weights(self):
        w, g = self.w, self.g
        return g["g1"], w["wqkv"], w["wo"], g["g2"], w["w1"], w["w2"]

    def forward(self, training=True):
        T.tsp_stack_forward(self.plan, self.x, *self.weights(), self.z, self.inputs if training else None,
                            self.saved if training else None, self.ws)
        T.tsp_sync_status(self.plan)
        return self.z.clone()

    def backward(self):
        s, n = self.shape, self.n
        dev = "cuda"
        self.dx = torch.empty(s.S, s.h, dtype=torch.bfloat16, device=dev)
        self.grads = {
            "dg1": [torch.empty(s.h, device=dev) for _ in range(n)],
            "dwqkv": [torch.empty(3 * s.h, s.h, device=dev) for _ in range(n)],
            "dwo": [torch.empty(s.h, s.h, device=dev) for _ in range(n)],
            "dg2": [torch.empty(s.h, device=dev) for _ in range(n)],
            "dw1": [torch.empty(s.ffn, s.h, device=dev) for _ in range(n)],
            "dw2": [torch.empty(s.h, s.ffn, device=dev) for _ in range(n)],
        }
        g = self.grads
        T.tsp_stack_backward(self.plan, self.dz, self.x, *self.weights(), self.inputs, self.saved, self.ws, self.dx,
                             g["dg1"], g["dwqkv"], g["dwo"], g["dg2"], g["dw1"], g["dw2"])
        T.tsp_sync_status(self.plan)
        return self.dx, g


def assert_close(name, gpu, ref, layers, report):
    assert np.all(np.isfinite(gpu)), name
    mx, mn = errors(gpu, ref)
    bmax, bmean = stack_bound_for(name, layers)
    report[name] = (mx, mn)
    assert mx <= bmax and mn <= bmean, f"{name}: max {mx:.3e} (bound {bmax:.1e}), mean {mn:.3e} (bound {bmean:.2e})"


def _oracle(st):
    inp, zig = st.inp, st.zig
    ws = [oracle_weights(lw) for lw in inp["layers"]]
    x = bits_to_f32(inp["x"][zig]).astype(np.float64)
    dz = bits_to_f32(inp["dy"][zig]).astype(np.float64)
    s = st.shape
    with OracleTimer("stack forward+backward", S=s.S, D=s.D, h=s.h, layers=st.n):
        z, caches = O.tsp_stack_forward(x, ws, s.heads, s.D)
        grads = O.tsp_stack_backward(dz, ws, caches)
    return z, grads


@pytest.mark.parametrize("shape,layers,seed", [
    (LayerShape(h=128, heads=4, ffn=512, S=256, D=2), 3, 0),
    (LayerShape(h=4096, heads=32, ffn=16384, S=4096, D=8), 2, 6),
], ids=["tiny_3layers", "7b_s4096_2layers"])
def test_stack_matches_the_oracle(shape, layers, seed):
    st = GpuStack(shape, layers, seed)
    z = host_f64(st.forward())
    dx, g = st.backward()
    zo, go = _oracle(st)
    report = {}
    assert_close("z", z, zo, layers, report)
    assert_close("dx", host_f64(dx), go[0]["dx"], layers, report)
    for i in range(layers):
        for k in GRADS:
            assert_close(k, host_f64(g[k][i]), go[i][k], layers, report)
    print(report)


def test_stack_equals_the_layer_calls_and_inference_forward():
    shape = LayerShape(h=128, heads=4, ffn=512, S=256, D=2)
    n = 3
    st = GpuStack(shape, n, 1)
    z = st.forward()
    dx, g = st.backward()
    z_inf = st.forward(training=False)
    assert torch.equal(z, z_inf)
    # by hand: every layer forward with its own saved buffer, then backward from the top
    ws_n, saved_n = T.tsp_workspace_size(st.plan, True)
    ws = torch.empty(ws_n, dtype=torch.uint8, device="cuda")
    g1, wqkv, wo, g2, w1, w2 = st.weights()
    acts, saves = [st.x], []
    for i in range(n):
        out = torch.empty_like(st.x)
        sv = torch.empty(saved_n, dtype=torch.uint8, device="cuda")
        T.tsp_layer_forward(st.plan, acts[-1], g1[i], wqkv[i], wo[i], g2[i], w1[i], w2[i], out, sv, ws)
        acts.append(out)
        saves.append(sv)
    assert torch.equal(acts[-1], z)
    grad = st.dz
    for i in reversed(range(n)):
        d = torch.empty_like(st.x)
        mine = {k: torch.empty_like(g[k][i]) for k in GRADS}
        T.tsp_layer_backward(st.plan, grad, acts[i], g1[i], wqkv[i], wo[i], g2[i], w1[i], w2[i], saves[i], ws, d,
                             mine["dg1"], mine["dwqkv"], mine["dwo"], mine["dg2"], mine["dw1"], mine["dw2"])
        for k in GRADS:
            assert torch.equal(mine[k], g[k][i]), (i, k)
        grad = d
    T.tsp_sync_status(st.plan)
    assert torch.equal(grad, dx)
