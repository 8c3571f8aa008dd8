"""tsp_plan's shape validation against the rules include/tsp.h states, on
randomly drawn shapes (hypothesis): each shape must give exactly the status
the documented rules assign, in their documented order."""

import pytest
from hypothesis import given, settings, strategies as st

import folded_tensor_sequence_map_b200 as T


def documented_status(h, heads, ffn, S, D):
    if h <= 0 or heads <= 0 or ffn <= 0 or S <= 0 or D <= 0:
        return "TSP_ERR_INVALID_ARG"
    if S % (2 * D) or heads % D or ffn % D or h % heads:
        return "TSP_ERR_INDIVISIBLE"
    dh = h // heads
    if dh not in (32, 64, 128):
        return "TSP_ERR_UNSUPPORTED"
    if h % 128 or S % 256 or (S // D) % 128 or ffn % 128 or (ffn // D) % 64:
        return "TSP_ERR_UNSUPPORTED"
    if S > (1 << 28) or heads * S * 32 + 255 > 2 ** 31 - 1:
        return "TSP_ERR_UNSUPPORTED"
    return "TSP_OK"


def plan_status(h, heads, ffn, S, D):
    try:
        T.tsp_plan(h, heads, ffn, S, D)
    except T.TSPError as e:
        return T.STATUS_NAMES[e.status]
    return "TSP_OK"


# shapes near the valid set: multiples that often satisfy the rules, plus noise
dims = st.one_of(st.sampled_from([128, 256, 512, 1024, 2048, 4096]), st.integers(-8, 5000))
head_counts = st.one_of(st.sampled_from([1, 2, 4, 8, 16, 32]), st.integers(-2, 70))
ffns = st.one_of(st.sampled_from([512, 1024, 2048, 4096, 16384]), st.integers(-8, 20000))
seqs = st.one_of(st.sampled_from([256, 512, 1024, 2048, 4096, 8192]), st.integers(-256, 20000))
ranks = st.one_of(st.sampled_from([1, 2, 4, 8, 16]), st.integers(-2, 40))


@settings(max_examples=400, deadline=None)
@given(h=dims, heads=head_counts, ffn=ffns, S=seqs, D=ranks)
def test_plan_status_follows_the_documented_rules(h, heads, ffn, S, D):
    assert plan_status(h, heads, ffn, S, D) == documented_status(h, heads, ffn, S, D)


@pytest.mark.parametrize("S,D", [(256, 1), (512, 2), (8192, 8), (4096, 16), (131072, 8)])
def test_accepted_shapes_follow_the_documented_rules(S, D):
    assert plan_status(4096, 32, 16384, S, D) == documented_status(4096, 32, 16384, S, D)
