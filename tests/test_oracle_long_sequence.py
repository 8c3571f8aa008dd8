"""Pin of the memory-bounded long-sequence evaluation (oracle/long_sequence.py)
to the plain oracle: on a small layer it must give what ``layer_forward``
followed by ``layer_backward`` gives, to fp64 rounding, with ragged row blocks
and with the heads spread over worker processes."""

import numpy as np
import pytest

import oracle as O


def _layer(rng, S, h, H, F_):
    x = rng.standard_normal((S, h))
    w = dict(
        wqkv=rng.standard_normal((3 * h, h)) * 0.3,
        wo=rng.standard_normal((h, h)) * 0.3,
        w1=rng.standard_normal((F_, h)) * 0.3,
        w2=rng.standard_normal((h, F_)) * 0.3,
        g1=1.0 + 0.3 * rng.standard_normal(h),
        g2=1.0 + 0.3 * rng.standard_normal(h),
    )
    return x, w, rng.standard_normal((S, h))


@pytest.mark.parametrize("row_block,workers", [(96, 1), (512, 2)])
def test_blocked_equals_plain_layer(row_block, workers):
    rng = np.random.default_rng(7)
    S, h, H, F_ = 384, 64, 4, 256
    x, w, dz = _layer(rng, S, h, H, F_)
    z, cache = O.layer_forward(x, w, H)
    ref = O.layer_backward(dz, w, H, cache)
    ref["z"] = z
    got = O.layer_forward_backward_blocked(x, w, dz, H, row_block=row_block, workers=workers)
    for k, v in ref.items():
        err = np.max(np.abs(got[k] - v)) / np.max(np.abs(v))
        assert err < 1e-12, (k, err)


def test_blocked_catches_a_wrong_head_split():
    # the head columns must be cut at dh: a layer whose heads are mislabelled
    # (H passed as 2 instead of 4) is a different function and must not match
    rng = np.random.default_rng(8)
    S, h, H, F_ = 256, 64, 4, 128
    x, w, dz = _layer(rng, S, h, H, F_)
    z, cache = O.layer_forward(x, w, H)
    got = O.layer_forward_backward_blocked(x, w, dz, 2, row_block=100)
    assert np.max(np.abs(got["z"] - z)) / np.max(np.abs(z)) > 1e-3
