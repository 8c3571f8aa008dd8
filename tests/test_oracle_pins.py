"""Pins of the fp64 oracle to things other than itself.

* integer invariants of the zigzag partition and of the shard schedules
  (closed forms, brute force, the chunk counts printed in the workload spec);
* PyTorch CPU fp64 library routines (rms_norm, gelu(tanh),
  scaled_dot_product_attention, linear) and autograd for the layer and its
  gradient;
* closed forms of attention on degenerate inputs;
* central finite differences of the folded layer;
* the folding identity: the folded layer equals the unsharded one for every D.
"""

import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_layer(rng, S, h, H, F_, wstd=0.3):
    x = rng.standard_normal((S, h))
    w = dict(
        wqkv=rng.standard_normal((3 * h, h)) * wstd,
        wo=rng.standard_normal((h, h)) * wstd,
        w1=rng.standard_normal((F_, h)) * wstd,
        w2=rng.standard_normal((h, F_)) * wstd,
        g1=1.0 + 0.3 * rng.standard_normal(h),
        g2=1.0 + 0.3 * rng.standard_normal(h),
    )
    return x, w


def _relerr(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


# ---------------------------------------------------------------------------
# zigzag partition
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("S,D", [(4, 1), (8, 2), (64, 4), (256, 2), (512, 8), (1024, 16)])
def test_zigzag_is_a_balanced_permutation(S, D):
    zig = O.zigzag_map(S, D)
    assert zig.shape == (D, S // D)
    assert np.array_equal(np.sort(zig.ravel()), np.arange(S))
    c = S // (2 * D)
    pairs = O.causal_pairs_per_rank(zig)
    # closed form: chunk j holds sum_{p=jc}^{jc+c-1} (p+1) = j c^2 + c(c+1)/2 pairs,
    # and chunks r and 2D-1-r add up to (2D-1) c^2 + c(c+1) for every rank.
    assert np.all(pairs == c * c * (2 * D - 1) + c * (c + 1))
    assert pairs.sum() == S * (S + 1) // 2


def test_zigzag_d1_is_identity():
    assert np.array_equal(O.zigzag_map(64, 1)[0], np.arange(64))


def test_zigzag_chunk_counts_match_workload_spec():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "zigzag_chunks.txt")) if l.strip() and l[0] != "#"]
    assert len(rows) == 4
    for S, D, nchunks, chunk in (map(int, r) for r in rows):
        zig = O.zigzag_map(S, D)
        # every rank holds exactly two runs of `chunk` consecutive positions,
        # each starting on a chunk boundary; together they are the n_chunks chunks
        starts = []
        for r in range(D):
            m = zig[r]
            assert len(m) == 2 * chunk
            for piece in (m[:chunk], m[chunk:]):
                assert np.all(np.diff(piece) == 1) and piece[0] % chunk == 0
                starts.append(int(piece[0]))
        assert sorted(starts) == [j * chunk for j in range(nchunks)]


def test_zigzag_tiny_brute_force_pairs():
    # every (q,k) pair with k <= q is owned by exactly one rank (the query's)
    S, D = 16, 2
    zig = O.zigzag_map(S, D)
    owner = np.empty(S, dtype=int)
    for r in range(D):
        owner[zig[r]] = r
    count = np.zeros(D, dtype=int)
    for q in range(S):
        for k in range(q + 1):
            count[owner[q]] += 1
    assert np.array_equal(count, O.causal_pairs_per_rank(zig))
    assert count[0] == count[1]


# ---------------------------------------------------------------------------
# shard schedules
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("D", [1, 2, 3, 4, 8, 16])
def test_schedules_are_latin(D):
    bc = O.shard_schedule(D, 0)
    ring = O.shard_schedule(D, 1)
    for r in range(D):
        assert sorted(bc[:, r]) == list(range(D))
        assert sorted(ring[:, r]) == list(range(D))
    for t in range(D):
        assert set(bc[t]) == {t}
        assert sorted(ring[t]) == list(range(D))  # every shard is somewhere at every step
        for r in range(D):
            assert ring[t, r] == (r + t) % D
            # point-to-point: what r holds at t+1 is what r+1 held at t
            if t + 1 < D:
                assert ring[t + 1, r] == ring[t, (r + 1) % D]


def test_schedule_rejects_bad_phase():
    with pytest.raises(ValueError):
        O.shard_schedule(4, 2)


# ---------------------------------------------------------------------------
# token-local pieces vs PyTorch library routines
# ---------------------------------------------------------------------------

def test_rmsnorm_matches_torch():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((7, 33)) * 3
    g = rng.standard_normal(33)
    out, rstd = O.rmsnorm(x, g)
    ref = F.rms_norm(torch.tensor(x), (33,), weight=torch.tensor(g), eps=1e-5).numpy()
    assert _relerr(out, ref) < 1e-13
    # gradient against autograd
    dout = rng.standard_normal((7, 33))
    xt = torch.tensor(x, requires_grad=True)
    gt = torch.tensor(g, requires_grad=True)
    F.rms_norm(xt, (33,), weight=gt, eps=1e-5).backward(torch.tensor(dout))
    dx, dg = O.rmsnorm_backward(dout, x, rstd, g)
    assert _relerr(dx, xt.grad.numpy()) < 1e-12
    assert _relerr(dg, gt.grad.numpy()) < 1e-12


def test_rmsnorm_special_case_constant_row():
    # a constant row c (|c| >> eps) normalises to sign(c) * g
    x = np.full((1, 16), -4.0)
    out, _ = O.rmsnorm(x, np.arange(16.0))
    assert np.allclose(out[0], -np.arange(16.0) / math.sqrt(1 + 1e-5 / 16))


def test_gelu_matches_torch():
    u = np.linspace(-8, 8, 2001)
    ut = torch.tensor(u, requires_grad=True)
    ref = F.gelu(ut, approximate="tanh")
    ref.backward(torch.ones_like(ut))
    assert _relerr(O.gelu_tanh(u), ref.detach().numpy()) < 1e-14
    assert _relerr(O.gelu_tanh_grad(u), ut.grad.numpy()) < 1e-13
    assert O.gelu_tanh(np.array([0.0]))[0] == 0.0
    assert abs(O.gelu_tanh_grad(np.array([0.0]))[0] - 0.5) < 1e-15


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def _sdpa(q, k, v, H):
    S, h = q.shape
    dh = h // H
    t = lambda a: torch.tensor(a).view(S, H, dh).transpose(0, 1)
    o = F.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=True)
    return o.transpose(0, 1).reshape(S, h)


def test_attention_matches_sdpa_global_order():
    rng = np.random.default_rng(2)
    S, H, dh = 300, 3, 16
    q, k, v = (rng.standard_normal((S, H * dh)) for _ in range(3))
    o, lse = O.causal_attention(q, k, v, np.arange(S), H)
    assert _relerr(o, _sdpa(q, k, v, H).numpy()) < 1e-12


def test_attention_matches_sdpa_zigzag_queries():
    rng = np.random.default_rng(3)
    S, D, H, dh = 128, 4, 2, 8
    q, k, v = (rng.standard_normal((S, H * dh)) for _ in range(3))
    ref = _sdpa(q, k, v, H).numpy()
    zig = O.zigzag_map(S, D)
    for r in range(D):
        o, _ = O.causal_attention(q[zig[r]], k, v, zig[r], H)
        assert _relerr(o, ref[zig[r]]) < 1e-12


def test_attention_closed_forms():
    # zero queries: every visible score is 0, so O_p = mean(V[0..p]) and
    # LSE_p = log(p + 1); the first query sees only key 0.
    rng = np.random.default_rng(4)
    S, H, dh = 50, 2, 4
    v = rng.standard_normal((S, H * dh))
    k = rng.standard_normal((S, H * dh))
    o, lse = O.causal_attention(np.zeros((S, H * dh)), k, v, np.arange(S), H)
    expect = np.cumsum(v, axis=0) / np.arange(1, S + 1)[:, None]
    assert _relerr(o, expect) < 1e-13
    assert np.allclose(lse, np.log(np.arange(1, S + 1))[None, :], rtol=0, atol=1e-13)
    q = rng.standard_normal((S, H * dh))
    o, _ = O.causal_attention(q, k, v, np.arange(S), H)
    assert np.allclose(o[0], v[0], rtol=0, atol=1e-15)


def test_attention_lse_matches_torch_logsumexp():
    rng = np.random.default_rng(5)
    S, H, dh = 40, 2, 8
    q, k, v = (rng.standard_normal((S, H * dh)) for _ in range(3))
    _, lse = O.causal_attention(q, k, v, np.arange(S), H)
    for n in range(H):
        c = slice(n * dh, (n + 1) * dh)
        s = torch.tensor(q[:, c]) @ torch.tensor(k[:, c]).T / math.sqrt(dh)
        s = s.masked_fill(torch.ones(S, S, dtype=torch.bool).triu(1), float("-inf"))
        assert _relerr(lse[n], torch.logsumexp(s, dim=1).numpy()) < 1e-13


def test_attention_backward_matches_autograd():
    rng = np.random.default_rng(6)
    S, H, dh = 96, 2, 8
    q, k, v, do = (rng.standard_normal((S, H * dh)) for _ in range(4))
    o, lse = O.causal_attention(q, k, v, np.arange(S), H)
    dq, dk, dv = O.causal_attention_backward(q, k, v, o, do, lse, np.arange(S), H)
    ts = [torch.tensor(a, requires_grad=True) for a in (q, k, v)]
    _sdpa_t = lambda a, b, c: F.scaled_dot_product_attention(
        *(x.view(S, H, dh).transpose(0, 1) for x in (a, b, c)), is_causal=True).transpose(0, 1).reshape(S, H * dh)
    _sdpa_t(*ts).backward(torch.tensor(do))
    for mine, t in zip((dq, dk, dv), ts):
        assert _relerr(mine, t.grad.numpy()) < 1e-11


# ---------------------------------------------------------------------------
# the whole layer vs a PyTorch fp64 composition of library routines
# ---------------------------------------------------------------------------

def torch_layer(x, w, H):
    S, h = x.shape
    dh = h // H
    a = F.rms_norm(x, (h,), weight=w["g1"], eps=1e-5)
    q, k, v = F.linear(a, w["wqkv"]).split(h, dim=1)
    heads = lambda t: t.view(S, H, dh).transpose(0, 1)
    o = F.scaled_dot_product_attention(heads(q), heads(k), heads(v), is_causal=True)
    y = x + F.linear(o.transpose(0, 1).reshape(S, h), w["wo"])
    b = F.rms_norm(y, (h,), weight=w["g2"], eps=1e-5)
    return y + F.linear(F.gelu(F.linear(b, w["w1"]), approximate="tanh"), w["w2"])


def _torch_grads(x, w, dz, H):
    xt = torch.tensor(x, requires_grad=True)
    wt = {k: torch.tensor(v, requires_grad=True) for k, v in w.items()}
    z = torch_layer(xt, wt, H)
    z.backward(torch.tensor(dz))
    g = {"d" + k: v.grad.numpy() for k, v in wt.items()}
    g["dx"] = xt.grad.numpy()
    return z.detach().numpy(), g


@pytest.mark.parametrize("S,h,H,F_", [(64, 32, 4, 64), (256, 128, 4, 512)])
def test_unsharded_layer_matches_torch(S, h, H, F_):
    rng = np.random.default_rng(7)
    x, w = _rand_layer(rng, S, h, H, F_, wstd=1.0 / math.sqrt(h))
    dz = rng.standard_normal((S, h))
    z, cache = O.layer_forward(x, w, H)
    grads = O.layer_backward(dz, w, H, cache)
    zt, gt = _torch_grads(x, w, dz, H)
    assert _relerr(z, zt) < 1e-12
    for key in ("dx", "dg1", "dwqkv", "dwo", "dg2", "dw1", "dw2"):
        assert _relerr(grads[key], gt[key]) < 1e-10, key


# ---------------------------------------------------------------------------
# folding identity and finite differences
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("D", [1, 2, 4, 8])
def test_folded_equals_unsharded(D):
    S, h, H, F_ = 64, 32, 8, 64
    rng = np.random.default_rng(8)
    x, w = _rand_layer(rng, S, h, H, F_, wstd=1.0 / math.sqrt(h))
    dz = rng.standard_normal((S, h))
    zg, cg = O.layer_forward(x, w, H)
    gg = O.layer_backward(dz, w, H, cg)
    perm = O.zigzag_map(S, D).ravel()
    zl, cl = O.tsp_layer_forward(x[perm], w, H, D)
    gl = O.tsp_layer_backward(dz[perm], w, cl)
    assert _relerr(zl, zg[perm]) < 1e-12
    assert _relerr(gl["dx"], gg["dx"][perm]) < 1e-12
    for key in ("dg1", "dwqkv", "dwo", "dg2", "dw1", "dw2"):
        assert _relerr(gl[key], gg[key]) < 1e-12, key


def test_forward_rows_match_full_forward():
    S, h, H, F_, D = 128, 32, 4, 64, 4
    rng = np.random.default_rng(9)
    x, w = _rand_layer(rng, S, h, H, F_, wstd=1.0 / math.sqrt(h))
    perm = O.zigzag_map(S, D).ravel()
    zl, _ = O.tsp_layer_forward(x[perm], w, H, D)
    rows = np.array([0, 5, 31, 32, 63, 64, 100, 127])
    assert _relerr(O.tsp_forward_rows(x[perm], w, H, D, rows), zl[rows]) < 1e-12


def test_folded_gradient_finite_differences():
    S, h, H, F_, D = 16, 8, 2, 16, 2
    rng = np.random.default_rng(10)
    x, w = _rand_layer(rng, S, h, H, F_, wstd=0.4)
    perm = O.zigzag_map(S, D).ravel()
    xl = x[perm]
    dz = rng.standard_normal((S, h))
    _, cache = O.tsp_layer_forward(xl, w, H, D)
    g = O.tsp_layer_backward(dz, w, cache)
    loss = lambda xx, ww: float(np.sum(O.tsp_layer_forward(xx, ww, H, D)[0] * dz))
    eps = 1e-6
    picks = np.random.default_rng(11)
    for name in ("x", "g1", "wqkv", "wo", "g2", "w1", "w2"):
        base = xl if name == "x" else w[name]
        for _ in range(6):
            idx = tuple(int(picks.integers(0, n)) for n in base.shape)
            plus, minus = base.copy(), base.copy()
            plus[idx] += eps
            minus[idx] -= eps
            if name == "x":
                fd = (loss(plus, w) - loss(minus, w)) / (2 * eps)
            else:
                fd = (loss(xl, {**w, name: plus}) - loss(xl, {**w, name: minus})) / (2 * eps)
            an = g["d" + name][idx]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, idx, fd, an)


def test_ring_partial_sums_stay_on_rank():
    # changing another rank's tokens must not change this rank's MLP partial sum
    # beyond what attention carries: with a D=2 layer whose attention output is
    # zeroed (Wo = 0), rank 0's output depends only on rank 0's tokens.
    S, h, H, F_, D = 32, 16, 2, 32, 2
    rng = np.random.default_rng(12)
    x, w = _rand_layer(rng, S, h, H, F_)
    w["wo"][:] = 0.0
    perm = O.zigzag_map(S, D).ravel()
    z1, _ = O.tsp_layer_forward(x[perm], w, H, D)
    x2 = x[perm].copy()
    x2[S // 2:] += 1.0  # rank 1's tokens
    z2, _ = O.tsp_layer_forward(x2, w, H, D)
    assert np.array_equal(z1[: S // 2], z2[: S // 2])
    assert not np.allclose(z1[S // 2:], z2[S // 2:])


# ---------------------------------------------------------------------------
# ring MLP on its own
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("D", [1, 2, 4, 8])
def test_ring_mlp_is_the_whole_mlp(D):
    """The ring's per-rank shard sums add up to the undivided MLP
    resid + GELU(b W1^T) W2^T on every row: a missing, repeated or misplaced
    shard, or a row block paired with the wrong rank, breaks the equality."""
    rng = np.random.default_rng(70 + D)
    S, h, F_ = 32 * D, 24, 8 * D
    b = rng.standard_normal((S, h))
    resid = rng.standard_normal((S, h))
    w1 = rng.standard_normal((F_, h)) * 0.3
    w2 = rng.standard_normal((h, F_)) * 0.3
    full = resid + O.gelu_tanh(b @ w1.T) @ w2.T
    assert _relerr(O.tsp_ring_mlp(b, w1, w2, resid, D), full) < 1e-12


def test_ring_mlp_matches_the_layer_oracle():
    """Given the layer's own normalised activations b and residual stream y,
    the standalone ring MLP reproduces the layer oracle's output z."""
    rng = np.random.default_rng(77)
    S, h, H, F_, D = 64, 16, 4, 32, 4
    x, w = _rand_layer(rng, S, h, H, F_)
    zl, cache = O.tsp_layer_forward(x[O.zigzag_map(S, D).ravel()], w, H, D)
    b = np.concatenate(cache["b"], axis=0)
    y = np.concatenate(cache["y"], axis=0)
    assert _relerr(O.tsp_ring_mlp(b, w["w1"], w["w2"], y, D), zl) < 1e-12


@pytest.mark.parametrize("H,dh,F,D", [(4, 32, 512, 2), (32, 128, 16384, 8), (16, 64, 4096, 16), (8, 32, 256, 1)])
def test_shards_partition_heads_and_ffn_units(H, dh, F, D):
    """Shard t of the attention weights is the contiguous block of heads
    [t H/D, (t+1) H/D) (their dh-wide column groups), and shard s of the MLP
    the units [s F/D, (s+1) F/D): over all shards, each column or unit
    exactly once, in order."""
    heads = [O.head_cols(t, H, D, dh) for t in range(D)]
    units = [O.ffn_units(s, F, D) for s in range(D)]
    assert np.array_equal(np.concatenate([np.arange(H * dh)[c] for c in heads]), np.arange(H * dh))
    assert np.array_equal(np.concatenate([np.arange(F)[u] for u in units]), np.arange(F))
    assert all((c.stop - c.start) == (H // D) * dh for c in heads)
    assert all((u.stop - u.start) == F // D for u in units)
