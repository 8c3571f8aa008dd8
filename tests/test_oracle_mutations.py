"""Plant plausible mistakes in the oracle (on the CPU, with monkeypatch) and
check that the pins in ``test_oracle_pins.py`` would catch each one: the
comparison against the PyTorch fp64 composition, or the integer invariants."""

import math

import numpy as np
import pytest

import oracle.tsp_oracle as T
from tests.test_oracle_pins import _relerr, _torch_grads, _rand_layer


def _layer_error():
    S, h, H, F_ = 64, 32, 4, 64
    rng = np.random.default_rng(21)
    x, w = _rand_layer(rng, S, h, H, F_, wstd=1.0 / math.sqrt(h))
    dz = rng.standard_normal((S, h))
    D = 2
    perm = T.zigzag_map(S, D).ravel()
    z, cache = T.tsp_layer_forward(x[perm], w, H, D)
    g = T.tsp_layer_backward(dz[perm], w, cache)
    zt, gt = _torch_grads(x, w, dz, H)
    errs = [_relerr(z, zt[perm]), _relerr(g["dx"], gt["dx"][perm])]
    errs += [_relerr(g[k], gt[k]) for k in ("dg1", "dwqkv", "dwo", "dg2", "dw1", "dw2")]
    return max(errs)


def test_unmutated_oracle_passes():
    assert _layer_error() < 1e-10


def _wrong_gelu_grad(u):
    t = np.tanh(T._GELU_K * (u + T._GELU_A * u ** 3))
    return 0.5 * (1.0 + t) + 0.5 * u * (1.0 - t * t) * T._GELU_K  # drops the cubic term's derivative


def _wrong_rms_bwd(dout, x, rstd, g):
    n = x * rstd[:, None]
    dn = dout * g[None, :]
    return rstd[:, None] * dn, np.sum(dout * n, axis=0)  # drops the projection term


def _wrong_attn_scale(q, k, v, qpos, H):
    return _orig_attn(q * math.sqrt(q.shape[1] // H) ** 0.5, k, v, qpos, H)


_orig_attn = T.causal_attention


def _strict_mask_attn(q, k, v, qpos, H):
    # excludes the diagonal (key < query) except for the first query
    return _orig_attn(q, k, v, np.maximum(qpos - 1, 0), H)


MUTATIONS = {
    "gelu_constant": ("_GELU_A", 0.047),
    "gelu_grad_term": ("gelu_tanh_grad", _wrong_gelu_grad),
    "rmsnorm_eps": ("EPS", 1e-3),
    "rmsnorm_bwd_term": ("rmsnorm_backward", _wrong_rms_bwd),
    "attention_scale": ("causal_attention", _wrong_attn_scale),
    "attention_mask": ("causal_attention", _strict_mask_attn),
    "ffn_shard_ignores_step": ("ffn_units", lambda s, F, D: slice(0, F // D)),
    "head_shard_ignores_step": ("head_cols", lambda t, H, D, dh: slice(0, (H // D) * dh)),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(monkeypatch, name):
    attr, value = MUTATIONS[name]
    monkeypatch.setattr(T, attr, value)
    if attr == "EPS":
        # default arguments captured EPS at definition time; patch the callers
        monkeypatch.setattr(T, "rmsnorm", lambda x, g, eps=1e-3: _rms(x, g, 1e-3))
    assert _layer_error() > 1e-6


def _rms(x, g, eps):
    rstd = 1.0 / np.sqrt(np.mean(x * x, axis=-1) + eps)
    return x * rstd[:, None] * g[None, :], rstd


def test_planted_ring_mistake_is_caught(monkeypatch):
    # a ring that skips a hop is no longer a Latin square
    def bad(D, phase):
        s = np.array([[(r + 2 * t) % D for r in range(D)] for t in range(D)])
        return s if phase == 1 else np.array([[t] * D for t in range(D)])
    monkeypatch.setattr(T, "shard_schedule", bad)
    ring = T.shard_schedule(4, 1)
    assert any(sorted(ring[:, r]) != list(range(4)) for r in range(4))


def test_planted_zigzag_mistake_is_caught(monkeypatch):
    # a contiguous (non-zigzag) split covers every token but is unbalanced
    monkeypatch.setattr(T, "zigzag_map", lambda S, D: np.arange(S).reshape(D, S // D))
    zig = T.zigzag_map(64, 4)
    pairs = T.causal_pairs_per_rank(zig)
    c = 64 // 8
    assert not np.all(pairs == c * c * 7 + c * (c + 1))


def _ring_mlp_error():
    """True when the ring-MLP pin fails."""
    from tests.test_oracle_pins import test_ring_mlp_is_the_whole_mlp
    try:
        for D in (2, 4):
            test_ring_mlp_is_the_whole_mlp(D)
    except AssertionError:
        return True
    return False


@pytest.mark.parametrize("mistake", ["shard_repeats", "rows_of_next_rank"])
def test_planted_ring_mlp_mistake_is_caught(monkeypatch, mistake):
    if mistake == "shard_repeats":
        # every step applies the rank's own shard again instead of rotating
        monkeypatch.setattr(T, "shard_schedule",
                            lambda D, phase: np.array([[r for r in range(D)] for _ in range(D)]))
    else:
        # each rank's partial sums are built from the next rank's rows
        orig = T.tsp_ring_mlp

        def shifted(b, w1, w2, resid, D):
            L = b.shape[0] // D
            return orig(np.roll(b, -L, axis=0), w1, w2, resid, D)
        monkeypatch.setattr(T, "tsp_ring_mlp", shifted)
        import oracle as O
        monkeypatch.setattr(O, "tsp_ring_mlp", shifted)
    assert _ring_mlp_error()


def test_unmutated_ring_mlp_passes():
    assert not _ring_mlp_error()
