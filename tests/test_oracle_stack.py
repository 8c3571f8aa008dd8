"""Pins of the oracle's stack of folded layers (``oracle.tsp_stack_*``).

The measured model of "Zyphra TSP folds TP+SP onto one GPU axis, 2.6x
throughput on 1,024 MI300Xs" (zubnet.ai, paragraph 1) is a stack of the
layer; between layers the tensors are bf16.  The stack's definition is the
composition of pinned layers, so the pins here check the composition itself:
* ``round_bf16`` equals PyTorch's float32 -> bfloat16 conversion (round to
  nearest, ties to even) and rounds exact ties to even;
* one layer is the layer oracle, call for call;
* a layer with Wo = W2 = 0 is the identity (z = x exactly, dx = dz exactly),
  so a stack ending in it equals the stack without it;
* central finite differences of <z, dz> (fp64, no interface rounding) match
  the stack's dx and a weight gradient of its lowest layer;
* with interface rounding, layer i+1 sees exactly round_bf16(z_i).
"""

import numpy as np
import pytest
import torch

import oracle as O
from synth_inputs import LayerShape, bits_to_f32, make_stack_inputs

SHAPE = LayerShape(h=64, heads=2, ffn=128, S=64, D=2)


def _weights(lw):
    w = {k: bits_to_f32(lw[k]).astype(np.float64) for k in ("wqkv", "wo", "w1", "w2")}
    w["g1"] = lw["g1"].astype(np.float64)
    w["g2"] = lw["g2"].astype(np.float64)
    return w


def _stack(layers, seed=7):
    inp = make_stack_inputs(SHAPE, layers, seed)
    zig = O.zigzag_map(SHAPE.S, SHAPE.D).ravel()
    x = bits_to_f32(inp["x"][zig]).astype(np.float64)
    dz = bits_to_f32(inp["dy"][zig]).astype(np.float64)
    return x, dz, [_weights(lw) for lw in inp["layers"]]


def test_round_bf16_is_round_to_nearest_even():
    rng = np.random.default_rng(0)
    x32 = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    want = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.round_bf16(x32.astype(np.float64)), want)
    # exact ties: 1 + 2^-8 sits halfway between 1 and 1 + 2^-7 (even: 1);
    # 1 + 3 * 2^-8 halfway between 1 + 2^-7 and 1 + 2^-6 (even: 1 + 2^-6)
    ties = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 0.0])
    assert np.array_equal(O.round_bf16(ties), [1.0, 1 + 2.0 ** -6, -1.0, 0.0])


def test_one_layer_is_the_layer():
    x, dz, ws = _stack(1)
    z, caches = O.tsp_stack_forward(x, ws, SHAPE.heads, SHAPE.D)
    z1, c1 = O.tsp_layer_forward(x, ws[0], SHAPE.heads, SHAPE.D)
    assert np.array_equal(z, z1)
    g = O.tsp_stack_backward(dz, ws, caches)[0]
    g1 = O.tsp_layer_backward(dz, ws[0], c1)
    for k in g1:
        assert np.array_equal(g[k], g1[k]), k


def test_zero_output_weights_make_an_identity_layer():
    x, dz, ws = _stack(2)
    ident = dict(ws[1])
    ident["wo"] = np.zeros_like(ident["wo"])
    ident["w2"] = np.zeros_like(ident["w2"])
    z, caches = O.tsp_stack_forward(x, [ws[0], ident], SHAPE.heads, SHAPE.D, round_interfaces=False)
    z0, c0 = O.tsp_layer_forward(x, ws[0], SHAPE.heads, SHAPE.D)
    assert np.array_equal(z, z0)
    g = O.tsp_stack_backward(dz, [ws[0], ident], caches, round_interfaces=False)
    assert np.array_equal(g[1]["dx"], dz)
    g0 = O.tsp_layer_backward(dz, ws[0], c0)
    for k in g0:
        assert np.array_equal(g[0][k], g0[k]), k


def test_finite_differences_through_two_layers():
    x, dz, ws = _stack(2)
    H, D = SHAPE.heads, SHAPE.D

    def f(xx, w0):
        z, _ = O.tsp_stack_forward(xx, [w0, ws[1]], H, D, round_interfaces=False)
        return float(np.sum(z * dz))

    _, caches = O.tsp_stack_forward(x, ws, H, D, round_interfaces=False)
    g = O.tsp_stack_backward(dz, ws, caches, round_interfaces=False)
    rng = np.random.default_rng(3)
    eps = 1e-5
    for _ in range(6):
        i, j = int(rng.integers(SHAPE.S)), int(rng.integers(SHAPE.h))
        xp, xm = x.copy(), x.copy()
        xp[i, j] += eps
        xm[i, j] -= eps
        fd = (f(xp, ws[0]) - f(xm, ws[0])) / (2 * eps)
        assert abs(fd - g[0]["dx"][i, j]) <= 1e-6 * max(1.0, abs(fd)), (i, j, fd, g[0]["dx"][i, j])
    for _ in range(4):
        i, j = int(rng.integers(SHAPE.h)), int(rng.integers(SHAPE.h))
        wp, wm = dict(ws[0]), dict(ws[0])
        wp["wo"] = ws[0]["wo"].copy()
        wm["wo"] = ws[0]["wo"].copy()
        wp["wo"][i, j] += eps
        wm["wo"][i, j] -= eps
        fd = (f(x, wp) - f(x, wm)) / (2 * eps)
        assert abs(fd - g[0]["dwo"][i, j]) <= 1e-6 * max(1.0, abs(fd)), (i, j, fd, g[0]["dwo"][i, j])


def test_interfaces_are_rounded_to_bf16():
    x, dz, ws = _stack(3)
    z, _ = O.tsp_stack_forward(x, ws, SHAPE.heads, SHAPE.D)
    # the input each upper layer sees is the rounded output of the one below
    cur = x
    for i in range(3):
        zi, _ = O.tsp_layer_forward(cur, ws[i], SHAPE.heads, SHAPE.D)
        if i < 2:
            cur = O.round_bf16(zi)
    assert np.array_equal(z, zi)
    zr, _ = O.tsp_stack_forward(x, ws, SHAPE.heads, SHAPE.D, round_interfaces=False)
    assert not np.array_equal(z, zr)
