"""Evidence for holding every tensor to the stated bounds (tests/tolerances.py).

A CPU model of the CUDA path's rounding placement (tests/precision_model.py)
is compared with the fp64 oracle at the 7B width (h=4096, 32 heads x 128,
FFN 16384) on a short sequence.  The test pins two facts:
* with fp16 tensor-core operands (the CUDA path) every output and gradient
  sits inside the stated bounds with room to spare (mean error at most 0.85
  of 2e-3, max error at most 0.5 of 1e-2), so the GPU tests can hold the
  kernels to them;
* with bf16 operands the same arithmetic misses the stated mean bound for the
  output and every gradient that passes through attention: the floor of that
  placement, not of the method.
"""

import numpy as np
import pytest

import oracle as O
from synth_inputs import LayerShape, bits_to_f32, make_layer_inputs
from tests.gpu_helpers import errors
from tests.precision_model import layer
from tests.tolerances import STATED


@pytest.fixture(scope="module")
def floors():
    shape = LayerShape(h=4096, heads=32, ffn=16384, S=512, D=2)
    inp = make_layer_inputs(shape, 1)
    w32 = {k: bits_to_f32(inp[k]) for k in ("wqkv", "wo", "w1", "w2")}
    w32["g1"], w32["g2"] = inp["g1"], inp["g2"]
    w64 = {k: v.astype(np.float64) for k, v in w32.items()}
    x, dy = bits_to_f32(inp["x"]), bits_to_f32(inp["dy"])
    z, cache = O.layer_forward(x.astype(np.float64), w64, shape.heads)
    ref = O.layer_backward(dy.astype(np.float64), w64, shape.heads, cache)
    ref["z"] = z
    out = {}
    for placement in ("f16", "bf16"):
        got = layer(x, w32, dy, shape.heads, placement)
        out[placement] = {k: errors(got[k].astype(np.float64), ref[k]) for k in ref}
    return out


def test_fp16_placement_meets_the_stated_bounds(floors):
    for name, (mx, mn) in floors["f16"].items():
        assert mn <= 0.85 * STATED[1] and mx <= 0.5 * STATED[0], (name, mx, mn)


def test_bf16_placement_misses_the_stated_mean_bound(floors):
    for name in ("z", "dx", "dg1", "dwqkv", "dwo"):
        assert floors["bf16"][name][1] > STATED[1], (name, floors["bf16"][name])
