"""Acceptance bounds of the GPU-vs-oracle comparisons.

Both bounds are relative to the oracle tensor:
    max|gpu - oracle|  <= B_max  * max|oracle|
    mean|gpu - oracle| <= B_mean * mean|oracle|

Every output and gradient is held to the stated bounds, B_max = 1e-2 and
B_mean = 2e-3.  They are within reach because every tensor-core operand the
layer computes itself is stored as fp16 (11-bit significand), not bf16: a CPU
model of this rounding placement (tests/test_precision_floor.py) puts the
error of each tensor at 0.2-0.8 of the stated mean bound at the 7B width,
while the same model with bf16 operands misses it for every tensor.

Intermediates (test-only views of the saved buffer) are compared at a looser
bound: U is kept in bf16 (it only feeds GELU'), and the others are single
roundings of values whose upstream error the outputs already bound.

A stack of L layers passes bf16 tensors between layers (its boundary dtype):
every layer's output activation and input gradient is rounded to bf16 once
more than in one layer.  Rounding to bf16 alone costs a mean relative error of
1.41e-3 (measured on the layer's z and dx, whose arithmetic adds only
0.05-0.2e-3 on top), and independent roundings add in quadrature.  Every
tensor of a stack sits downstream of up to L such roundings: z and every
activation above the first layer in the forward, and every gradient of a
lower layer through the gradient handed down to it (its dg and dW are linear
in that gradient).  So the stack's mean bound is sqrt(L) times the stated
one for every tensor (max bound unchanged); measured on the 7B layer at
S=4096 with 2 layers: dx 2.39e-3 and layer 0's dg1 2.18e-3 mean (bound
2.83e-3), the top layer's tensors at the single layer's errors.
"""

import math

STATED = (1e-2, 2e-3)

# Intermediates (test-only views of the saved buffer).
INTERMEDIATE = (2e-2, 1e-2)


def bound_for(name: str):
    if name.startswith("mid."):
        return INTERMEDIATE
    return STATED


def stack_bound_for(name: str, layers: int):
    """Bounds of a tensor of an L-layer stack (see above)."""
    bmax, bmean = bound_for(name)
    return bmax, bmean * math.sqrt(layers)
