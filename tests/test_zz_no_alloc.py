"""The RMSNorm backward entry point that allocates nothing.

Some callers cannot allocate device memory (cudaMalloc is not allowed where
they run, or they have no memory pool to take scratch from).  For them the
library keeps the scratch of this step (partial sums of the gain gradient) in
a device array of its own.  This test runs the tiny layer's forward and
backward through the ordinary entry points, then calls the no-allocation entry
point twice in a row on the same intermediates the layer's last backward stage
used, and checks that both calls reproduce the layer's dx and dg1.  The layer
keeps those intermediates times a power of two 2^k (its scaled gradient
domain); the test multiplies them by 2^-k first, which is exact in fp32, so
the results must agree bit for bit.  It sits in a file of its own, collected
last.
"""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

import folded_tensor_sequence_map_b200 as T
from synth_inputs import WORKLOADS, make_layer_inputs
from tests.gpu_helpers import GpuLayer, assert_close, host_f64


def test_noalloc_matches_layer_backward_twice():
    shape, seed = WORKLOADS["tiny"]
    inp = make_layer_inputs(shape, seed)
    L = GpuLayer(shape, inp, training=True)
    L.forward()
    g = L.backward()
    S, h = shape.S, shape.h
    da = L.saved_view("ws.da", (S, h), torch.float32)
    dy = L.saved_view("ws.dy", (S, h), torch.float32)
    rstd1 = L.saved_view("rstd1", (S,), torch.float32)
    unscale = L.saved_view("ws.gscales", (2,), torch.float32)[0]
    da = (da * unscale).contiguous()
    dy = (dy * unscale).contiguous()
    ref_dx, ref_dg = host_f64(g["dx"]), host_f64(g["dg1"])
    for _ in range(2):
        dx = torch.full((S, h), float("nan"), dtype=torch.bfloat16, device="cuda")
        dg = torch.full((h,), float("nan"), dtype=torch.float32, device="cuda")
        T.tsp_rmsnorm_backward_noalloc(da, L.x, rstd1, L.g1, dy, dx, dg, S, h)
        torch.cuda.synchronize()
        got_dx, got_dg = host_f64(dx), host_f64(dg)
        assert_close("dx", got_dx, ref_dx)
        assert_close("dg1", got_dg, ref_dg)
        # same kernel, same inputs: the results are identical
        assert np.array_equal(got_dx, ref_dx) and np.array_equal(got_dg, ref_dg)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # one 64-row block more than the 4,194,304-float array holds at h = 4096;
    # the size check comes before anything is enqueued
    h = 4096
    rows = 64 * (4194304 // h + 1)
    t = torch.empty(16, device="cuda")
    p = t.data_ptr()
    status = T._lib.tsp_rmsnorm_backward_noalloc(p, p, p, p, p, p, p, rows, h, None)
    assert T.STATUS_NAMES[status] == "TSP_ERR_UNSUPPORTED"
