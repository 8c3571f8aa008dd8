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
"""

STATED = (1e-2, 2e-3)

# Intermediates (test-only views of the saved buffer).
INTERMEDIATE = (2e-2, 1e-2)


def bound_for(name: str):
    if name.startswith("mid."):
        return INTERMEDIATE
    return STATED
