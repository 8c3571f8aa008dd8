"""Tiny layer (h=128, 4 heads x 32, FFN 512, S=256, D=2): the CUDA path against
the oracle, element by element, for the output, every gradient and every
saved intermediate."""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import oracle as O
from synth_inputs import WORKLOADS, bits_to_f32, make_layer_inputs
from tests.gpu_helpers import GpuLayer, assert_close, host_f64, oracle_weights

LOG2E = 1.4426950408889634


@pytest.fixture(scope="module")
def tiny():
    shape, seed = WORKLOADS["tiny"]
    inp = make_layer_inputs(shape, seed)
    layer = GpuLayer(shape, inp, training=True)
    z = host_f64(layer.forward())
    grads = {k: host_f64(v) for k, v in layer.backward().items()}
    zig = layer.zig
    w = oracle_weights(inp)
    xl = bits_to_f32(inp["x"][zig]).astype(np.float64)
    dyl = bits_to_f32(inp["dy"][zig]).astype(np.float64)
    zo, cache = O.tsp_layer_forward(xl, w, shape.heads, shape.D)
    go = O.tsp_layer_backward(dyl, w, cache)
    return dict(shape=shape, layer=layer, z=z, grads=grads, zo=zo, cache=cache, go=go)


def test_forward_intermediates(tiny):
    s, L, c = tiny["shape"], tiny["layer"], tiny["cache"]
    S, h, F, H = s.S, s.h, s.ffn, s.heads
    cat = lambda k: np.concatenate(c[k], axis=0)
    views = {
        "a": (cat("a"), (S, h), torch.float16),
        "q": (cat("Q"), (S, h), torch.float16),
        "k": (c["Kg"], (S, h), torch.float16),
        "v": (c["Vg"], (S, h), torch.float16),
        "o": (cat("O"), (S, h), torch.float16),
        "y": (cat("y"), (S, h), torch.float32),
        "b": (cat("b"), (S, h), torch.float16),
        "u": (cat("U"), (S, F), torch.bfloat16),
    }
    for name, (ref, shp, dt) in views.items():
        got = host_f64(L.saved_view(name, shp, dt))
        assert_close("mid." + name, got, ref)
    lse = host_f64(L.saved_view("lse", (H, S), torch.float32))
    lse_ref = np.concatenate(c["lse"], axis=1) * LOG2E
    assert np.abs(lse - lse_ref).max() < 2e-2


def test_forward_output(tiny):
    assert_close("z", tiny["z"], tiny["zo"])


@pytest.mark.parametrize("name", ["dx", "dg1", "dwqkv", "dwo", "dg2", "dw1", "dw2"])
def test_backward_outputs(tiny, name):
    assert_close(name, tiny["grads"][name], tiny["go"][name])


def test_repeat_is_bitwise_deterministic(tiny):
    L = tiny["layer"]
    z2 = host_f64(L.forward())
    g2 = {k: host_f64(v) for k, v in L.backward().items()}
    assert np.array_equal(z2, tiny["z"])
    for k in g2:
        assert np.array_equal(g2[k], tiny["grads"][k]), k


def test_head_size_64_layer_against_oracle():
    # dh = 64 (h=256, 4 heads x 64, FFN 1024, S=512, D=2): the single-atom
    # 128-byte-swizzle path of the attention kernels, every output and gradient
    from synth_inputs import LayerShape

    shape = LayerShape(h=256, heads=4, ffn=1024, S=512, D=2)
    inp = make_layer_inputs(shape, 6)
    layer = GpuLayer(shape, inp, training=True)
    z = host_f64(layer.forward())
    grads = {k: host_f64(v) for k, v in layer.backward().items()}
    w = oracle_weights(inp)
    zig = layer.zig
    zo, cache = O.tsp_layer_forward(bits_to_f32(inp["x"][zig]).astype(np.float64), w, shape.heads, shape.D)
    go = O.tsp_layer_backward(bits_to_f32(inp["dy"][zig]).astype(np.float64), w, cache)
    assert_close("z", z, zo)
    for k in go:
        assert_close(k, grads[k], go[k])


@pytest.mark.parametrize("S,D,heads", [(512, 1, 4), (512, 4, 4), (1024, 2, 4), (1024, 8, 8)])
def test_head_size_128_layer_against_oracle(S, D, heads):
    # dh = 128 (heads x 128, FFN 4h): the single-pass attention backward with
    # its ordered dQ sum, at zigzag chunks of 64 to 512 rows
    from synth_inputs import LayerShape

    shape = LayerShape(h=128 * heads, heads=heads, ffn=512 * heads, S=S, D=D)
    inp = make_layer_inputs(shape, 7)
    layer = GpuLayer(shape, inp, training=True)
    z = host_f64(layer.forward())
    grads = {k: host_f64(v) for k, v in layer.backward().items()}
    w = oracle_weights(inp)
    zig = layer.zig
    zo, cache = O.tsp_layer_forward(bits_to_f32(inp["x"][zig]).astype(np.float64), w, shape.heads, shape.D)
    go = O.tsp_layer_backward(bits_to_f32(inp["dy"][zig]).astype(np.float64), w, cache)
    assert_close("z", z, zo)
    for k in go:
        assert_close(k, grads[k], go[k])
    # the same call again gives the same bits (the dQ sum is order-fixed)
    layer.forward()
    g2 = {k: host_f64(v) for k, v in layer.backward().items()}
    for k in g2:
        assert np.array_equal(g2[k], grads[k]), k
