"""Device-side pieces checked on their own: the bounded wait that every
kernel uses (it gives up and reports instead of hanging) and the attention
forward's polynomial exp2."""

import pytest
import torch

pytestmark = pytest.mark.gpu

import folded_tensor_sequence_map_b200 as T


def test_bounded_wait_gives_up_and_reports_timeout():
    plan = T.tsp_plan(128, 4, 512, 256, 2)
    result = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    T.tsp_test_wait_timeout(plan, 2_000_000, result)  # ~1 ms at the boost clock
    with pytest.raises(T.TSPError) as e:
        T.tsp_sync_status(plan)
    assert T.STATUS_NAMES[e.value.status] == "TSP_ERR_TIMEOUT"
    assert int(result.item()) == 0
    T.tsp_sync_status(plan)  # the flag was cleared by the report


def test_polynomial_exp2_error_bound():
    """The attention forward's exp2 on the FMA pipe (Cody-Waite split into
    round(x) and a fraction in [-1/2, 1/2], degree-5 minimax polynomial)
    stays within 2.5e-7 relative error of 2^x over the arguments the softmax
    produces (the fit's bound in fp32 is 2.13e-7; the split and the 2^n
    scaling are exact), as close as the hardware approximation it replaces;
    arguments at or below -127, -inf included, give 0 or a denormal."""
    import numpy as np

    rng = np.random.default_rng(5)
    x = np.concatenate([np.linspace(-126.0, 16.0, 1 << 22), rng.uniform(-30.0, 16.0, 1 << 20),
                        np.arange(-126, 17, dtype=np.float64), np.arange(-126, 16) + 0.5]).astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    ys = {}
    for which in (0, 1):
        y = torch.empty_like(xd)
        T.tsp_test_exp2(xd, y, which)
        ys[which] = y.cpu().numpy().astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = {w: float(np.abs(ys[w] / ref - 1.0).max()) for w in ys}
    print(f"max relative error: polynomial {rel[0]:.3e}, hardware approximation {rel[1]:.3e}")
    assert rel[0] <= 2.5e-7
    low = torch.tensor([-np.inf, -1e30, -1000.0, -127.0, -126.75, -126.5000001], dtype=torch.float32, device="cuda")
    y = torch.empty_like(low)
    T.tsp_test_exp2(low, y, 0)
    y = y.cpu().numpy()
    assert np.all(y >= 0.0) and np.all(y < 2.0 ** -126)
