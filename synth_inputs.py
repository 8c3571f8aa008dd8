"""Seeded synthetic inputs for the folded TSP decoder layer.

This module is shared by the tests, the benchmark and the oracle's callers.  It
holds none of the layer's arithmetic: it only draws numbers and rounds them to
bf16, so both the CUDA path and the fp64 oracle start from bit-identical
inputs.

Recipe (one 7B-shaped or tiny pre-RMSNorm decoder layer, batch 1):

* ``rng = np.random.default_rng(seed)`` (PCG64), ``standard_normal`` drawn in
  float32, in this order: x ``[S, h]``, Wqkv ``[3h, h]``, Wo ``[h, h]``,
  W1 ``[F, h]``, W2 ``[h, F]``, then (when asked for) dY ``[S, h]``.
* Weights are the draw times 0.02 (computed in float32); x and dY are N(0, 1).
* Every array is rounded to bf16 with round-to-nearest-even.
* RMSNorm gains g1, g2 are ones (float32).
* x and dY are drawn in GLOBAL token order; putting them in rank-major zigzag
  order is the caller's job (with the library's or the oracle's zigzag map),
  so a sweep over D sees identical tokens.

Wqkv rows are the Q heads 0..H-1 (dh rows each), then the K heads, then the V
heads; every weight uses the ``[out, in]`` row-major layout of a linear layer.
"""

from __future__ import annotations

import hashlib
from dataclasses import dataclass

import numpy as np

WEIGHT_STD = 0.02


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even); return the
    16-bit patterns as uint16.  Inputs here are finite normal draws."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to the float32 values they encode."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class LayerShape:
    """Shape of one decoder layer plus its folded-axis size."""

    h: int
    heads: int
    ffn: int
    S: int
    D: int

    @property
    def dh(self) -> int:
        return self.h // self.heads


# Named workloads: (shape, seed).  Sizes follow the layer specification of
# each configuration; the 7B shape is h=4096, 32 heads, FFN 16384.
WORKLOADS = {
    "tiny": (LayerShape(h=128, heads=4, ffn=512, S=256, D=2), 0),
    "7b_s8k": (LayerShape(h=4096, heads=32, ffn=16384, S=8192, D=8), 1),
    "7b_s32k": (LayerShape(h=4096, heads=32, ffn=16384, S=32768, D=8), 2),
    "7b_s32k_bwd": (LayerShape(h=4096, heads=32, ffn=16384, S=32768, D=8), 3),
    "7b_s128k": (LayerShape(h=4096, heads=32, ffn=16384, S=131072, D=8), 4),
}


def make_layer_inputs(shape: LayerShape, seed: int, with_dy: bool = True) -> dict:
    """Draw one layer's inputs.  Returns a dict of uint16 bf16 bit arrays
    (x, wqkv, wo, w1, w2 and optionally dy) plus float32 gains g1, g2."""
    h, F, S = shape.h, shape.ffn, shape.S
    rng = np.random.default_rng(seed)
    out = {}
    out["x"] = bf16_bits(rng.standard_normal((S, h), dtype=np.float32))
    for name, shp in (("wqkv", (3 * h, h)), ("wo", (h, h)), ("w1", (F, h)), ("w2", (h, F))):
        w = rng.standard_normal(shp, dtype=np.float32)
        w *= np.float32(WEIGHT_STD)
        out[name] = bf16_bits(w)
    if with_dy:
        out["dy"] = bf16_bits(rng.standard_normal((S, h), dtype=np.float32))
    out["g1"] = np.ones(h, dtype=np.float32)
    out["g2"] = np.ones(h, dtype=np.float32)
    return out


def make_layer_weights(shape: LayerShape, seed: int) -> dict:
    """Draw one layer's weights alone: Wqkv, Wo, W1, W2 from
    ``default_rng(seed)`` in that order (times 0.02, rounded to bf16), gains
    ones.  Used for the layers of a stack, each with its own seed."""
    h, F = shape.h, shape.ffn
    rng = np.random.default_rng(seed)
    out = {}
    for name, shp in (("wqkv", (3 * h, h)), ("wo", (h, h)), ("w1", (F, h)), ("w2", (h, F))):
        w = rng.standard_normal(shp, dtype=np.float32)
        w *= np.float32(WEIGHT_STD)
        out[name] = bf16_bits(w)
    out["g1"] = np.ones(h, dtype=np.float32)
    out["g2"] = np.ones(h, dtype=np.float32)
    return out


def make_stack_inputs(shape: LayerShape, layers: int, seed: int) -> dict:
    """Inputs of a stack of ``layers`` layers: x and dY as make_layer_inputs
    draws them for ``seed``, and layer i's weights from
    make_layer_weights(shape, seed * 1000 + 1 + i).  Returns dict(x, dy,
    layers=[weights of layer 0, ...])."""
    inp = make_layer_inputs(shape, seed)
    return dict(x=inp["x"], dy=inp["dy"],
                layers=[make_layer_weights(shape, seed * 1000 + 1 + i) for i in range(layers)])


def sample_rows(S: int, n: int, seed: int) -> np.ndarray:
    """Seeded sample of ``n`` distinct row indices in [0, S) that always
    includes the first and the last row; sorted ascending."""
    rng = np.random.default_rng(seed + 1000)
    rows = rng.choice(S, size=min(n, S), replace=False)
    rows[0] = 0
    if len(rows) > 1:
        rows[1] = S - 1
    return np.unique(rows)


def input_hash(inp: dict) -> str:
    """sha256 of the bf16 bit patterns of x, Wqkv, Wo, W1, W2 and dY, in that
    order: identifies the inputs that a stored expected value belongs to."""
    hsh = hashlib.sha256()
    for k in ("x", "wqkv", "wo", "w1", "w2", "dy"):
        hsh.update(np.ascontiguousarray(inp[k]).tobytes())
    return hsh.hexdigest()
