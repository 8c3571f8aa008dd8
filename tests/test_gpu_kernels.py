"""The bounded wait that every kernel uses: it gives up and reports instead of
hanging."""

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
