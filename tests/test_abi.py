"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol the headers declare, and its integer outputs (zigzag map, shard
schedules) match the oracle bit for bit; argument errors are reported."""

import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O
import folded_tensor_sequence_map_b200 as T
import folded_tensor_sequence_map_b200.tsp as TT

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for hdr in ("tsp.h", "tsp_testing.h"):
        src = open(os.path.join(ROOT, "include", hdr)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"\b(tsp_[a-z0-9_]+)\s*\(", src))
    return names


def test_library_exports_every_declared_symbol():
    import ctypes

    declared = _declared_functions()
    assert {"tsp_plan", "tsp_zigzag_map", "tsp_layer_forward", "tsp_layer_backward"} <= declared
    lib = ctypes.CDLL(T.LIB_PATH)
    for name in sorted(declared):
        assert hasattr(lib, name), name
    assert declared == set(T.EXPORTED)


@pytest.mark.parametrize("h,H,F,S,D", [(128, 4, 512, 256, 2), (4096, 32, 16384, 8192, 8),
                                       (4096, 32, 16384, 131072, 8), (4096, 32, 16384, 131072, 16),
                                       (4096, 32, 16384, 131072, 1), (256, 4, 1024, 2048, 4)])
def test_zigzag_and_schedules_match_oracle(h, H, F, S, D):
    p = T.tsp_plan(h, H, F, S, D)
    assert np.array_equal(T.tsp_zigzag_map(p), O.zigzag_map(S, D).ravel())
    for phase in (0, 1):
        assert np.array_equal(T.tsp_shard_schedule(p, phase), O.shard_schedule(D, phase))


@pytest.mark.parametrize("h,H,F,S,D", [(128, 4, 512, 256, 2), (4096, 32, 16384, 8192, 8), (2048, 16, 4096, 4096, 16),
                                       (256, 4, 1024, 2048, 1), (4096, 32, 16384, 131072, 8)])
def test_next_visible_matches_zigzag_scan(h, H, F, S, D):
    """The dK/dV kernel's walk over query steps: the first 64-row local step at
    or after `start` holding a row whose position (oracle zigzag map) is at
    least kv0, found here by scanning every step."""
    p = T.tsp_plan(h, H, F, S, D)
    nq = S // 64
    step_max = O.zigzag_map(S, D).ravel().reshape(nq, 64).max(axis=1)
    rng = np.random.default_rng(S + D)
    kv0s = np.unique(np.concatenate([[0, 1, 63, 64, 127, S // 2, S - 128, S - 64, S - 1],
                                     rng.integers(0, S, 60), np.arange(0, S, max(128, S // 256))]))
    for kv0 in kv0s:
        vis = np.nonzero(step_max >= kv0)[0]
        starts = np.unique(np.concatenate([[0, 1, nq - 1, nq], rng.integers(0, nq + 1, 10), vis[:2], vis[-2:],
                                           np.maximum(vis[:2] - 1, 0)]).astype(int))
        for st in starts:
            later = vis[vis >= st]
            want = int(later[0]) if len(later) else nq
            assert T.tsp_test_next_visible(p, int(st), int(kv0)) == want, (S, D, kv0, st)
    for bad in ((-1, 0), (nq + 1, 0), (0, -1), (0, S)):
        with pytest.raises(T.TSPError):
            T.tsp_test_next_visible(p, *bad)


@pytest.mark.parametrize("h,H,F,S,D", [(128, 4, 512, 256, 2), (4096, 32, 16384, 8192, 8), (2048, 16, 4096, 4096, 16),
                                       (256, 4, 1024, 2048, 1), (4096, 32, 16384, 32768, 8),
                                       (4096, 32, 16384, 131072, 8)])
def test_step_walk_visits_exactly_the_visible_steps(h, H, F, S, D):
    """The dK/dV kernel's walk for a key tile at kv0 visits, in ascending
    order and once each, exactly the 64-row local steps holding a row at a
    position >= kv0 (oracle zigzag map)."""
    p = T.tsp_plan(h, H, F, S, D)
    step_max = O.zigzag_map(S, D).ravel().reshape(S // 64, 64).max(axis=1)
    rng = np.random.default_rng(S * 3 + D)
    tiles = np.unique(np.concatenate([[0, 1, S // 256, S // 128 - 1], rng.integers(0, S // 128, 24)]))
    for kt in tiles:
        kv0 = int(kt) * 128
        want = np.nonzero(step_max >= kv0)[0]
        assert np.array_equal(T.tsp_test_step_walk(p, kv0), want), (S, D, kv0)


@pytest.mark.parametrize("h,H,F,S,D", [(128, 4, 512, 256, 2), (4096, 32, 16384, 8192, 8), (2048, 16, 4096, 4096, 16),
                                       (256, 4, 1024, 2048, 1), (4096, 32, 16384, 131072, 8)])
def test_descending_walk_is_a_prefix_of_one_order(h, H, F, S, D):
    """The single-pass backward's walk for a key tile at kv0 visits exactly the
    64-row local steps holding a row at a position >= kv0 (oracle zigzag map),
    once each, in strictly descending order of position, and is a prefix of
    the walk for kv0 = 0 (so key tiles walked at the same time touch the same
    query rows)."""
    p = T.tsp_plan(h, H, F, S, D)
    nq = S // 64
    zig = O.zigzag_map(S, D).ravel().reshape(nq, 64)
    step_max, step_min = zig.max(axis=1), zig.min(axis=1)
    full = T.tsp_test_step_walk(p, 0, descending=True)
    assert np.array_equal(np.sort(full), np.arange(nq))
    assert np.all(np.diff(step_min[full]) < 0) and np.all(step_max[full][1:] < step_min[full][:-1])
    rng = np.random.default_rng(S * 5 + D)
    tiles = np.unique(np.concatenate([[0, 1, S // 256, S // 128 - 1], rng.integers(0, S // 128, 24)]))
    for kt in tiles:
        kv0 = int(kt) * 128
        walk = T.tsp_test_step_walk(p, kv0, descending=True)
        assert np.array_equal(np.sort(walk), np.nonzero(step_max >= kv0)[0]), (S, D, kv0)
        assert np.array_equal(walk, full[:len(walk)]), (S, D, kv0)


@pytest.mark.parametrize("h,H,F,S,D", [(256, 2, 1024, 1024, 2), (512, 4, 2048, 2048, 4),
                                       (4096, 32, 16384, 32768, 8)])
def test_rank_walk_and_order_keep_to_the_rank_rows(h, H, F, S, D):
    """One rank's share of the single-pass backward: its walk for a key tile is
    the whole-layer walk with every step outside the rank's L local rows left
    out (same order), and its work order holds each (key tile, head) whose
    walk is non-empty exactly once: the key tiles at or below the highest
    position of the rank's rows (oracle zigzag map)."""
    p = T.tsp_plan(h, H, F, S, D)
    L, nq = S // D, S // 64
    zig = O.zigzag_map(S, D).ravel()
    rng = np.random.default_rng(S + 7 * D)
    tiles = np.unique(np.concatenate([[0, 1, S // 256, S // 128 - 1], rng.integers(0, S // 128, 16)]))
    for r in range(D):
        mine = (np.arange(nq) >= r * L // 64) & (np.arange(nq) < (r + 1) * L // 64)
        for kt in tiles:
            full = T.tsp_test_step_walk(p, int(kt) * 128, descending=True)
            walk = T.tsp_test_step_walk_rank(p, r, int(kt) * 128)
            assert np.array_equal(walk, full[mine[full]]), (S, D, r, kt)
        top = zig[r * L:(r + 1) * L].max()
        seen = np.array([kt * H + hd for kt in range(S // 128) if kt * 128 <= top for hd in range(H)])
        order = T.tsp_test_rank_kv_order(p, r, 148)
        assert np.array_equal(np.sort(order), seen), (S, D, r)
        for kt in np.unique(order // H):  # no item without steps
            assert len(T.tsp_test_step_walk_rank(p, r, int(kt) * 128)) > 0
        beyond = (int(top) // 128 + 1) * 128
        if beyond < S:
            assert len(T.tsp_test_step_walk_rank(p, r, beyond)) == 0
    assert T.STATUS_NAMES[TT._lib.tsp_test_step_walk_rank(p.handle, D, 0, None, 0, ctypes.byref(ctypes.c_int()))] \
        == "TSP_ERR_INVALID_ARG"


def test_rank_backward_checks_arguments_before_enqueueing():
    """tsp_rank_backward_attn / _qkv refuse a head size other than 128, a rank
    outside [0, D), a NULL or a misaligned pointer before anything runs."""
    p = T.tsp_plan(256, 2, 1024, 1024, 2)
    V = ctypes.c_void_p
    lib = TT._lib
    st = lambda rc: T.STATUS_NAMES[rc]
    good = [V(0x10000 * (i + 1)) for i in range(12)]
    attn = lambda plan, rank, args: st(lib.tsp_rank_backward_attn(plan.handle, rank, *args[:12], V(0)))
    qkv = lambda plan, rank, args: st(lib.tsp_rank_backward_qkv(plan.handle, rank, *args[:9], V(0)))
    for f in (attn, qkv):
        assert f(p, 2, good) == "TSP_ERR_INVALID_ARG" and f(p, -1, good) == "TSP_ERR_INVALID_ARG"
        bad = list(good)
        bad[4] = V(0)
        assert f(p, 0, bad) == "TSP_ERR_INVALID_ARG"
        bad = list(good)
        bad[1] = V(0x20008)
        assert f(p, 1, bad) == "TSP_ERR_ALIGNMENT"
        assert f(T.tsp_plan(128, 4, 512, 1024, 2), 0, good) == "TSP_ERR_UNSUPPORTED"  # head size 32
    assert T.tsp_rank_backward_workspace_size(p) > 0


def _start_spread(cost, G):
    """Largest gap, over the rounds of G items, between the first and the last
    start time of a round's items when CTA i runs items i, i + G, ... at one
    unit of time per unit of cost."""
    n = len(cost)
    t = np.zeros(G)
    worst = 0
    for r0 in range(0, n, G):
        c = cost[r0:r0 + G]
        worst = max(worst, t[:len(c)].max() - t[:len(c)].min())
        t[:len(c)] += c
    return worst


@pytest.mark.parametrize("G", [1, 7, 148])
@pytest.mark.parametrize("S", [4096, 32768, 131072])
def test_uploaded_work_orders_pair_long_and_short_items(G, S):
    """The orders the plan uploads for G SMs: every item once; within a head
    the j-th longest item pairs with the j-th shortest, a wave of G pairs laid
    out as the long items then the short ones.  So CTA i (items i, i + G, ...)
    runs one pair per wave, every pair has the same length up to rounding, and
    the CTAs start each round's items within one wave's length differences of
    each other: with the head-major host order the starts drift apart by a
    whole walk."""
    h, H, F, D = 4096, 32, 16384, 8
    p = T.tsp_plan(h, H, F, S, D)
    zig = O.zigzag_map(S, D).ravel()
    steps = np.array([(zig.reshape(S // 64, 64).max(axis=1) >= kt * 128).sum() for kt in range(S // 128)])
    for name, width in (("fwd_order", 2), ("kv_order", 1)):
        base = T.tsp_test_tables(p, name).reshape(-1, width)
        up = T.tsp_test_work_order(p, name, G).reshape(-1, width)
        assert np.array_equal(np.sort(up[:, 0]), np.sort(base[:, 0])), (name, G)
        if width == 2:
            assert np.array_equal(up[np.argsort(up[:, 0])], base[np.argsort(base[:, 0])])
        cost = up[:, 1] if width == 2 else steps[up[:, 0] // H]
        n = len(cost)
        npairs = n // 2
        for w0 in range(0, npairs, G):
            w1 = min(w0 + G, npairs)
            longs, shorts = cost[2 * w0:2 * w0 + (w1 - w0)], cost[2 * w0 + (w1 - w0):2 * w1]
            heads_l = up[2 * w0:2 * w0 + (w1 - w0), 0] % H
            heads_s = up[2 * w0 + (w1 - w0):2 * w1, 0] % H
            assert np.array_equal(heads_l, heads_s)
            assert np.all(longs >= shorts)
            pair = longs + shorts
            assert pair.max() - pair.min() <= 2, (name, G, w0)
        if G == 148 and S >= 32768:
            base_cost = base[:, 1] if width == 2 else steps[base[:, 0] // H]
            paired, plain = _start_spread(cost, G), _start_spread(base_cost, G)
            # a round's starts differ by at most the long items' length range
            # of a wave; without pairing they drift by a whole walk and more
            assert paired <= cost.max() - cost.min() and paired * 4 < plain, (name, paired, plain)
    with pytest.raises(T.TSPError):
        T.tsp_test_work_order(p, "kv_order", 0)
    with pytest.raises(T.TSPError):
        T.tsp_test_work_order(p, "inv", G)


@pytest.mark.parametrize("h,H,F,S,D", [(128, 4, 512, 256, 2), (4096, 32, 16384, 8192, 8), (2048, 16, 4096, 4096, 16),
                                       (256, 4, 1024, 2048, 1), (4096, 32, 16384, 32768, 8)])
def test_kernel_tables_match_the_zigzag_map(h, H, F, S, D):
    """The tables the plan uploads, rebuilt from the oracle's zigzag map: the
    inverse map, each 128-row tile's largest position, and three attention
    work orders.  Each order covers every item once, head-major, longest
    first within a head."""
    p = T.tsp_plan(h, H, F, S, D)
    zig = O.zigzag_map(S, D).ravel()
    inv = T.tsp_test_tables(p, "inv")
    assert np.array_equal(zig[inv], np.arange(S))
    qmax = T.tsp_test_tables(p, "qtile_maxpos")
    assert np.array_equal(qmax, zig.reshape(S // 128, 128).max(axis=1))

    def head_major_longest_first(items, cost):
        heads = items % H
        assert np.all(np.diff(heads) >= 0)
        for hd in range(H):
            c = cost[heads == hd]
            assert np.all(np.diff(c) <= 0)

    fwd = T.tsp_test_tables(p, "fwd_order").reshape(-1, 2)
    items, nkv = fwd[:, 0], fwd[:, 1]
    assert np.array_equal(np.sort(items), np.arange((S // 256) * H))
    block_max = zig.reshape(S // 256, 256).max(axis=1)
    assert np.array_equal(nkv, block_max[items // H] // 128 + 1)
    head_major_longest_first(items, nkv)

    kv = T.tsp_test_tables(p, "kv_order")
    assert np.array_equal(np.sort(kv), np.arange((S // 128) * H))
    seen_by = np.array([(qmax >= kt * 128).sum() for kt in range(S // 128)])
    head_major_longest_first(kv, seen_by[kv // H])

    q = T.tsp_test_tables(p, "q_order")
    assert np.array_equal(np.sort(q), np.arange((S // 128) * H))
    head_major_longest_first(q, qmax[q // H])

    n = ctypes.c_int64()
    rc = TT._lib.tsp_test_tables(p.handle, 7, None, 0, ctypes.byref(n))
    assert T.STATUS_NAMES[rc] == "TSP_ERR_INVALID_ARG"


def test_stack_checks_arguments_before_enqueueing():
    """tsp_stack_forward / tsp_stack_backward refuse a bad layer count, a NULL
    in a weight or gradient array, or a misaligned pointer before anything
    runs (the addresses are never dereferenced); the workspace sizes follow
    the layer's: one layer's saved buffer, the layer scratch plus three
    activations, and layers-1 kept inputs."""
    h, H, F, S, D = 128, 4, 512, 256, 2
    p = T.tsp_plan(h, H, F, S, D)
    ws1, saved1 = T.tsp_workspace_size(p, True)
    ws_inf, _ = T.tsp_workspace_size(p, False)
    act = S * h * 2
    for n in (1, 3, 32):
        ws, saved, inputs = T.tsp_stack_workspace_size(p, n)
        assert saved == saved1 and inputs == (n - 1) * act and ws == max(ws1, ws_inf) + 3 * act
    V = ctypes.c_void_p
    arr = lambda n, base=0x100000: (V * n)(*[base + 0x1000 * i for i in range(n)])
    lib = TT._lib
    st = lambda rc: T.STATUS_NAMES[rc]
    good = dict(x=0x20000, z=0x30000, inputs=0x40000, saved=0x50000, ws=0x60000)
    fwd = lambda n, arrs, **kw: lib.tsp_stack_forward(p.handle, n, V(kw.get("x", good["x"])),
                                                        *[ctypes.cast(a, V) for a in arrs], V(kw.get("z", good["z"])),
                                                        V(good["inputs"]), V(good["saved"]), V(good["ws"]), V(0))
    six = [arr(3) for _ in range(6)]
    assert st(fwd(0, six)) == "TSP_ERR_INVALID_ARG"
    holey = [arr(3) for _ in range(6)]
    holey[2][1] = None
    assert st(fwd(3, holey)) == "TSP_ERR_INVALID_ARG"
    assert st(fwd(3, six, x=good["x"] + 8)) == "TSP_ERR_ALIGNMENT"
    bwd = lambda n, arrs, grads, dx=0x70000: lib.tsp_stack_backward(
        p.handle, n, V(0x80000), V(good["x"]), *[ctypes.cast(a, V) for a in arrs], V(good["inputs"]),
        V(good["saved"]), V(good["ws"]), V(dx), *[ctypes.cast(a, V) for a in grads], V(0))
    grads = [arr(3, 0x900000) for _ in range(6)]
    assert st(bwd(0, six, grads)) == "TSP_ERR_INVALID_ARG"
    gholey = [arr(3, 0x900000) for _ in range(6)]
    gholey[5][2] = None
    assert st(bwd(3, six, gholey)) == "TSP_ERR_INVALID_ARG"
    assert st(bwd(3, six, grads, dx=0x70008)) == "TSP_ERR_ALIGNMENT"


def test_rank_forward_checks_arguments_before_enqueueing():
    """tsp_rank_forward_qkv / _out refuse a rank outside [0, D), a NULL or a
    misaligned pointer, and a rank size L that is not a multiple of 256 (the
    attention's query blocks), before anything runs."""
    p = T.tsp_plan(128, 4, 512, 1024, 2)
    V = ctypes.c_void_p
    lib = TT._lib
    st = lambda rc: T.STATUS_NAMES[rc]
    good = [V(0x10000 * (i + 1)) for i in range(9)]
    qkv = lambda rank, args: st(lib.tsp_rank_forward_qkv(p.handle, rank, *args[:6], V(0)))
    out = lambda rank, args: st(lib.tsp_rank_forward_out(p.handle, rank, *args[:9], V(0)))
    assert qkv(2, good) == "TSP_ERR_INVALID_ARG" and qkv(-1, good) == "TSP_ERR_INVALID_ARG"
    assert out(2, good) == "TSP_ERR_INVALID_ARG"
    bad = list(good)
    bad[3] = V(0)
    assert qkv(0, bad) == "TSP_ERR_INVALID_ARG" and out(0, bad) == "TSP_ERR_INVALID_ARG"
    bad = list(good)
    bad[2] = V(0x30008)
    assert qkv(1, bad) == "TSP_ERR_ALIGNMENT" and out(1, bad) == "TSP_ERR_ALIGNMENT"
    small = T.tsp_plan(128, 4, 512, 256, 2)  # L = 128
    assert st(lib.tsp_rank_forward_qkv(small.handle, 0, *good[:6], V(0))) == "TSP_ERR_UNSUPPORTED"
    assert T.tsp_rank_workspace_size(p) > 0


def test_prefill_checks_arguments_before_enqueueing():
    """tsp_layer_prefill refuses a NULL or misaligned pointer before it touches
    the device (the addresses below are never dereferenced)."""
    p = T.tsp_plan(128, 4, 512, 256, 2)
    good = [0x10000 * (i + 1) for i in range(11)]
    for i in range(11):
        args = list(good)
        args[i] = None
        with pytest.raises(T.TSPError) as e:
            T.tsp_layer_prefill(p, *args, stream=0)
        assert T.STATUS_NAMES[e.value.status] == "TSP_ERR_INVALID_ARG"
        args = list(good)
        args[i] += 8
        with pytest.raises(T.TSPError) as e:
            T.tsp_layer_prefill(p, *args, stream=0)
        assert T.STATUS_NAMES[e.value.status] == "TSP_ERR_ALIGNMENT"


def test_ring_mlp_workspace_and_argument_checks():
    """Scratch for U and G ([S][F] each), the fp16 copies of b [S][h], W1 and W2
    [F][h] each, and the scales (256-byte aligned pieces); NULL or misaligned
    pointers are refused before anything is enqueued."""
    p = T.tsp_plan(128, 4, 512, 256, 2)
    S, h, F = 256, 128, 512
    assert T.tsp_ring_mlp_workspace_size(p) >= 2 * S * F * 2 + S * h * 2 + 2 * F * h * 2 + 64 * 4
    good = [0x10000 * (i + 1) for i in range(6)]
    for i in range(6):
        args = list(good)
        args[i] = None
        with pytest.raises(T.TSPError) as e:
            T.tsp_ring_mlp_forward(p, *args, stream=0)
        assert T.STATUS_NAMES[e.value.status] == "TSP_ERR_INVALID_ARG"
        args = list(good)
        args[i] += 4
        with pytest.raises(T.TSPError) as e:
            T.tsp_ring_mlp_forward(p, *args, stream=0)
        assert T.STATUS_NAMES[e.value.status] == "TSP_ERR_ALIGNMENT"


def test_flops_formula_matches_workload_figures():
    # algorithmic FLOPs of the forward: 24 S h^2 + 2 h S (S+1) for the 7B shape
    for S, expect in ((256, None), (8192, 3.848e12), (32768, 2.199e13), (131072, 1.935e14)):
        if expect is None:
            p = T.tsp_plan(128, 4, 512, S, 2)
            assert T.tsp_layer_flops(p, False) == 2 * S * (4 * 128**2 + 2 * 128 * 512) + 2 * 128 * S * (S + 1)
            continue
        p = T.tsp_plan(4096, 32, 16384, S, 8)
        assert abs(T.tsp_layer_flops(p, False) / expect - 1) < 1e-3
        assert T.tsp_layer_flops(p, True) == 2 * T.tsp_layer_flops(p, False)


def test_workspace_sizes_cover_the_layout():
    p = T.tsp_plan(128, 4, 512, 256, 2)
    ws_t, saved_t = T.tsp_workspace_size(p, True)
    ws_i, saved_i = T.tsp_workspace_size(p, False)
    S, h, F, H = 256, 128, 512, 4
    assert saved_i == 0 and ws_i == saved_t
    weights = (3 * h * h + h * h + 2 * F * h) * 2
    assert saved_t >= S * h * 2 * 6 + S * h * 4 + S * F * 2 * 2 + H * S * 4 + 2 * S * 4 + weights
    assert ws_t >= S * F * 2 + S * h * (4 + 4 + 2 + 2 + 4 + 2) + S * 3 * h * 2
    names = ["rstd1", "a", "q", "k", "v", "o", "lse", "y", "rstd2", "b", "u", "g", "wqkv_h", "wo_h", "w1_h",
             "w2_h", "scales"]
    offs = [T.tsp_test_buffer_offset(p, n) for n in names]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs) and offs[-1] < saved_t
    with pytest.raises(T.TSPError):
        T.tsp_test_buffer_offset(p, "nope")


@pytest.mark.parametrize("args,status", [
    ((128, 4, 512, 250, 2), "TSP_ERR_INDIVISIBLE"),
    ((128, 3, 512, 256, 2), "TSP_ERR_INDIVISIBLE"),
    ((128, 4, 511, 256, 2), "TSP_ERR_INDIVISIBLE"),
    ((96, 4, 512, 256, 2), "TSP_ERR_UNSUPPORTED"),      # dh = 24
    ((128, 4, 512, 128, 1), "TSP_ERR_UNSUPPORTED"),     # S % 256
    ((128, 4, 512, 256, 4), "TSP_ERR_UNSUPPORTED"),     # S/D = 64 tokens per rank
    ((0, 4, 512, 256, 2), "TSP_ERR_INVALID_ARG"),
    ((128, 4, 512, 0, 2), "TSP_ERR_INVALID_ARG"),      # no tokens
    ((128, 4, 512, 256, 0), "TSP_ERR_INVALID_ARG"),    # no ranks
    ((128, 0, 512, 256, 2), "TSP_ERR_INVALID_ARG"),
    ((128, 4, 0, 256, 2), "TSP_ERR_INVALID_ARG"),
    ((128, 4, 512, -256, 2), "TSP_ERR_INVALID_ARG"),
    ((128, 4, 512, 256, -2), "TSP_ERR_INVALID_ARG"),
    ((128, 4, 512, 384, 2), "TSP_ERR_UNSUPPORTED"),     # ragged: S % 256
    ((128, 4, 448, 256, 2), "TSP_ERR_UNSUPPORTED"),     # ffn % 128
    ((128, 4, 512, 768, 3), "TSP_ERR_INDIVISIBLE"),     # heads % D
])
def test_plan_rejects_bad_shapes(args, status):
    with pytest.raises(T.TSPError) as e:
        T.tsp_plan(*args)
    assert T.STATUS_NAMES[e.value.status] == status
    assert T.tsp_status_string(e.value.status) == status


def test_plan_size_limit_of_the_thread_numbering():
    """heads * S may not exceed 67,108,856 (one warp per token and head,
    numbered with 32-bit integers); the largest S below it is accepted."""
    ok = T.tsp_plan(128, 4, 512, (1 << 24) - 256, 2)
    assert ok.S == (1 << 24) - 256
    del ok
    with pytest.raises(T.TSPError) as e:
        T.tsp_plan(128, 4, 512, 1 << 24, 2)
    assert T.STATUS_NAMES[e.value.status] == "TSP_ERR_UNSUPPORTED"
    with pytest.raises(T.TSPError) as e:
        T.tsp_plan(4096, 32, 16384, 1 << 21, 8)
    assert T.STATUS_NAMES[e.value.status] == "TSP_ERR_UNSUPPORTED"


def test_bad_phase_is_rejected():
    p = T.tsp_plan(128, 4, 512, 256, 2)
    with pytest.raises(T.TSPError):
        T.tsp_shard_schedule(p, 2)


def test_exp2_polynomial_coefficients_are_the_fit():
    """The polynomial in the attention forward's exp2 is the one the Remez
    fit produces (degree 5, coefficients rounded to fp32), and the fit's
    relative error in fp32 is what the kernel's comment and GPU test state."""
    from folded_tensor_sequence_map_b200.csrc import fit_exp2 as F

    src = open(os.path.join(ROOT, "folded_tensor_sequence_map_b200", "csrc", "attn_fwd.cu")).read()
    body = src[src.index("float exp2_poly(float x)"):]
    body = body[:body.index("\n}\n")]
    used = [float.fromhex(h) for h in re.findall(r"(0x1\.[0-9a-f]+p[-+]\d+)f", body)]
    c = F.remez_relative(5).astype(np.float32)
    # Horner from the top coefficient: c5, c4 in the first fma, then c3 .. c0
    assert used == [float(c[5]), float(c[4]), float(c[3]), float(c[2]), float(c[1]), float(c[0])]
    grid = np.linspace(F.LO, F.HI, 200001)
    err = np.abs(F.horner_f32(c, grid).astype(np.float64) / np.exp2(grid.astype(np.float32).astype(np.float64)) - 1)
    assert err.max() <= 2.2e-7


@pytest.mark.parametrize("S", [32768, 131072])
def test_rank_orders_keep_the_ctas_in_step(S):
    """One rank's backward order for 148 SMs is the one of two that keeps the
    CTAs' start times closer together (CTA i runs items i, i + G, ...; cost =
    the rank's query steps that see the key tile, from the oracle's zigzag
    map): paired in waves like the layer's, or head-major with the longest
    items first.  Paired, each wave's long and short items come from the same
    heads and each long item is at least as long as its partner.  Ranks 0 and
    D/2-1 take the pairs (their spread is several times smaller); rank D-1,
    whose key tiles mostly share one cost, does at least as well as
    head-major."""
    h, H, F, D, G = 4096, 32, 16384, 8, 148
    p = T.tsp_plan(h, H, F, S, D)
    zig = O.zigzag_map(S, D).ravel()
    L = S // D
    for r in (0, D // 2 - 1, D - 1):
        smax = zig[r * L:(r + 1) * L].reshape(L // 64, 64).max(axis=1)
        cost_kt = np.array([(smax >= kt * 128).sum() for kt in range(S // 128)])
        up = T.tsp_test_rank_kv_order(p, r, G)
        cost = cost_kt[up // H]
        hm = np.array(sorted(up, key=lambda it: (it % H, -cost_kt[it // H], it // H)))
        spread, spread_hm = _start_spread(cost, G), _start_spread(cost_kt[hm // H], G)
        assert spread <= spread_hm, (S, r, spread, spread_hm)
        if r < D - 1:
            assert 2 * spread < spread_hm, (S, r, spread, spread_hm)
        if np.array_equal(up, hm):
            continue
        npairs = len(up) // 2
        for w0 in range(0, npairs, G):
            w1 = min(w0 + G, npairs)
            nw = w1 - w0
            longs, shorts = cost[2 * w0:2 * w0 + nw], cost[2 * w0 + nw:2 * w1]
            assert np.array_equal(up[2 * w0:2 * w0 + nw] % H, up[2 * w0 + nw:2 * w1] % H), (S, r, w0)
            assert np.all(longs >= shorts), (S, r, w0)
