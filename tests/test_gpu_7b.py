"""7B-shaped layer (h=4096, 32 heads x 128, FFN 16384) against the oracle.

* S=8192, D=8: forward and forward+backward, every element.
* S=32768, D=8: forward+backward, every element of every output and gradient
  (seed 3; z on every row).
* D sweep {1, 2, 4, 8, 16} at S=4096: every D against one run of the
  unsharded oracle (the inputs are drawn in global order, so every D sees the
  same tokens and the same exact result, permuted).
* S=131072, D=8, in the launch configuration the benchmark times, against
  fp64-oracle values stored by tests/golden/make_s131072_backward.py (which
  calls only the oracle): z and dx on the seeded sample of 512 rows (rows 0 and
  S-1 included), dg1 and dg2 whole, and 65,536 seeded entries of each weight
  gradient.  As a supplement the folding identity is checked GPU against GPU:
  the gradients at D=8 equal those at D=1 and D=16.
"""

import os

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import oracle as O
from synth_inputs import WORKLOADS, LayerShape, bits_to_f32, input_hash, make_layer_inputs, sample_rows
from tests.gpu_helpers import GpuLayer, OracleTimer, assert_close, errors, host_f64, oracle_weights
from tests.tolerances import bound_for

GRADS = ("dx", "dg1", "dwqkv", "dwo", "dg2", "dw1", "dw2")
GOLDEN_128K = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "s131072_d8_seed4.npz")


def _run(shape, seed, training):
    inp = make_layer_inputs(shape, seed, with_dy=training)
    layer = GpuLayer(shape, inp, training=training)
    z = host_f64(layer.forward())
    grads = {k: host_f64(v) for k, v in layer.backward().items()} if training else None
    return inp, layer.zig, z, grads


def _oracle(shape, inp, zig, training):
    w = oracle_weights(inp)
    x = bits_to_f32(inp["x"][zig]).astype(np.float64)
    meta = dict(S=shape.S, D=shape.D, h=shape.h, heads=shape.heads, ffn=shape.ffn)
    with OracleTimer("folded forward", **meta):
        z, cache = O.tsp_layer_forward(x, w, shape.heads, shape.D)
    g = None
    if training:
        with OracleTimer("folded backward", **meta):
            g = O.tsp_layer_backward(bits_to_f32(inp["dy"][zig]).astype(np.float64), w, cache)
    del cache
    return z, g


@pytest.mark.parametrize("training", [False, True])
def test_7b_s8192(training):
    shape, seed = WORKLOADS["7b_s8k"]
    inp, zig, z, grads = _run(shape, seed, training)
    zo, go = _oracle(shape, inp, zig, training)
    report = {}
    assert_close("z", z, zo, report)
    if training:
        for k in GRADS:
            assert_close(k, grads[k], go[k], report)
    print(report)


@pytest.mark.slow
def test_7b_s32768_forward_backward():
    shape, seed = WORKLOADS["7b_s32k_bwd"]
    inp, zig, z, grads = _run(shape, seed, True)
    zo, go = _oracle(shape, inp, zig, True)
    report = {}
    assert_close("z", z, zo, report)
    for k in GRADS:
        assert_close(k, grads[k], go[k], report)
    print(report)


@pytest.fixture(scope="module")
def sweep_oracle():
    shape = LayerShape(h=4096, heads=32, ffn=16384, S=4096, D=1)
    inp = make_layer_inputs(shape, 5)
    w = oracle_weights(inp)
    zg, cache = O.layer_forward(bits_to_f32(inp["x"]).astype(np.float64), w, shape.heads)
    gg = O.layer_backward(bits_to_f32(inp["dy"]).astype(np.float64), w, shape.heads, cache)
    return zg, gg


@pytest.mark.parametrize("D", [1, 2, 4, 8, 16])
def test_d_sweep_against_unsharded_oracle(D, sweep_oracle):
    zg, gg = sweep_oracle
    shape = LayerShape(h=4096, heads=32, ffn=16384, S=4096, D=D)
    inp, zig, z, grads = _run(shape, 5, True)
    assert_close("z", z, zg[zig])
    assert_close("dx", grads["dx"], gg["dx"][zig])
    for k in GRADS[1:]:
        assert_close(k, grads[k], gg[k])


@pytest.fixture(scope="module")
def s128k():
    shape, seed = WORKLOADS["7b_s128k"]
    inp, zig, z, grads = _run(shape, seed, True)
    return shape, seed, inp, zig, z, grads


def test_7b_s131072_against_stored_oracle_values(s128k):
    shape, seed, inp, zig, z, grads = s128k
    gold = np.load(GOLDEN_128K)
    assert str(gold["input_sha256"]) == input_hash(inp), "stored values belong to other inputs"
    rows = gold["rows"]
    assert np.array_equal(rows, sample_rows(shape.S, 512, seed)) and 0 in rows and shape.S - 1 in rows
    assert np.array_equal(gold["pos"], zig[rows])
    report = {}
    assert_close("z", z[rows], gold["z"].astype(np.float64), report)
    assert_close("dx", grads["dx"][rows], gold["dx"].astype(np.float64), report)
    for k in ("dg1", "dg2"):
        assert_close(k, grads[k], gold[k].astype(np.float64), report)
    for k in ("dwqkv", "dwo", "dw1", "dw2"):
        assert_close(k, grads[k].ravel()[gold[k + "_idx"]], gold[k + "_val"].astype(np.float64), report)
    print(report)


@pytest.mark.parametrize("D2", [1, 16])
def test_7b_s131072_backward_folding_identity(s128k, D2):
    shape, seed, inp, zig, z, grads = s128k
    other = LayerShape(h=shape.h, heads=shape.heads, ffn=shape.ffn, S=shape.S, D=D2)
    layer = GpuLayer(other, inp, training=True)
    z2 = host_f64(layer.forward())
    g2 = {k: host_f64(v) for k, v in layer.backward().items()}
    # un-permute both to global order
    inv8 = np.empty_like(zig)
    inv8[zig] = np.arange(len(zig))
    inv2 = np.empty_like(layer.zig)
    inv2[layer.zig] = np.arange(len(zig))
    for name, a, b in [("z", z[inv8], z2[inv2]), ("dx", grads["dx"][inv8], g2["dx"][inv2])] + \
            [(k, grads[k], g2[k]) for k in GRADS[1:]]:
        mx, mn = errors(a, b)
        # two computations of the same quantity: each is within its bound of the
        # exact value, so they agree within twice that bound
        bmax, bmean = bound_for(name)
        assert mx <= 2 * bmax and mn <= 2 * bmean, (name, mx, mn)
