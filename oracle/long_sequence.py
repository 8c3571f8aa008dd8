"""Memory-bounded evaluation of the unsharded layer's forward and backward for
long sequences (test infrastructure only, like the rest of ``oracle``).

At S = 131072 and the 7B width one fp64 [S, h] activation is 4.3 GB and the
MLP pre-activation [S, F] is 17 GB, so the plain ``layer_forward`` /
``layer_backward`` pair does not fit a 62 GB host.  This module evaluates the
same arithmetic with the same primitives of ``tsp_oracle`` (``rmsnorm``,
``rmsnorm_backward``, ``gelu_tanh``, ``gelu_tanh_grad``, ``causal_attention``,
``causal_attention_backward``), and changes only how the work is cut so that
memory stays bounded:

* token-local steps (the RMSNorms, the projections, the MLP and its
  gradient) run on blocks of consecutive token rows: every one of them is a
  function of its own row, and the weight gradients, which sum over rows, are
  sums of the blocks' pieces;
* attention runs one head at a time: heads do not interact until the
  out-projection, and ``causal_attention`` of one head is the multi-head call
  restricted to that head's dh columns.  Heads are spread over worker
  processes; the per-head operands and results pass through .npy files.

No result depends on the cut except through fp64 summation order.  The
equality with ``layer_forward`` + ``layer_backward`` is pinned on the CPU.

Layer ([Z1], [Z2] as cited in ``tsp_oracle``): pre-RMSNorm, causal softmax
attention, out-projection and residual, pre-RMSNorm, GELU(tanh) MLP and
residual; the folding identity makes the unsharded layer the folded one's
result in global token order.
"""

from __future__ import annotations

import multiprocessing as mp
import os
import shutil
import tempfile

import numpy as np

from .tsp_oracle import (EPS, causal_attention, causal_attention_backward, gelu_tanh, gelu_tanh_grad, rmsnorm,
                         rmsnorm_backward)


def _head_forward(args):
    d, n = args
    q = np.load(os.path.join(d, f"q{n}.npy"), mmap_mode="r")
    k = np.load(os.path.join(d, f"k{n}.npy"), mmap_mode="r")
    v = np.load(os.path.join(d, f"v{n}.npy"), mmap_mode="r")
    S = q.shape[0]
    o, lse = causal_attention(np.asarray(q), np.asarray(k), np.asarray(v), np.arange(S), 1)
    np.save(os.path.join(d, f"o{n}.npy"), o)
    np.save(os.path.join(d, f"lse{n}.npy"), lse[0])
    return n


def _head_backward(args):
    d, n = args
    ld = lambda name: np.asarray(np.load(os.path.join(d, f"{name}{n}.npy"), mmap_mode="r"))
    q, k, v, o, do, lse = ld("q"), ld("k"), ld("v"), ld("o"), ld("do"), ld("lse")
    S = q.shape[0]
    dq, dk, dv = causal_attention_backward(q, k, v, o, do, lse[None, :], np.arange(S), 1)
    np.save(os.path.join(d, f"dq{n}.npy"), dq)
    np.save(os.path.join(d, f"dk{n}.npy"), dk)
    np.save(os.path.join(d, f"dv{n}.npy"), dv)
    return n


def _per_head(fn, d, H, workers):
    jobs = [(d, n) for n in range(H)]
    if workers <= 1:
        for j in jobs:
            fn(j)
        return
    # spawn: the workers start clean whatever the parent holds
    with mp.get_context("spawn").Pool(workers, initializer=_single_thread_blas) as pool:
        for _ in pool.imap_unordered(fn, jobs):
            pass


def _single_thread_blas():
    try:
        from threadpoolctl import threadpool_limits

        threadpool_limits(1)
    except ImportError:  # pragma: no cover
        pass


def layer_forward_backward_blocked(x, w, dz, H, *, row_block=4096, workers=1, scratch=None, log=None):
    """Forward and exact backward of the unsharded layer (global token order)
    on fp64 inputs, with the memory bounds described in the module docstring.

    ``x``, ``dz``: [S, h]; ``w``: wqkv [3h, h], wo [h, h], w1 [F, h], w2 [h, F],
    g1, g2 [h].  Returns a dict with z, dx [S, h] and dg1, dwqkv, dwo, dg2,
    dw1, dw2, the same quantities as ``layer_forward`` followed by
    ``layer_backward``."""
    say = log or (lambda *_: None)
    x = np.asarray(x, dtype=np.float64)
    dz = np.asarray(dz, dtype=np.float64)
    w = {k: np.asarray(v, dtype=np.float64) for k, v in w.items()}
    S, h = x.shape
    dh = h // H
    F = w["w1"].shape[0]
    own = scratch is None
    d = tempfile.mkdtemp(prefix="tsp_oracle_") if own else scratch
    os.makedirs(d, exist_ok=True)
    blocks = [slice(i, min(i + row_block, S)) for i in range(0, S, row_block)]
    try:
        # RMSNorm1 and the Q/K/V projections, per row block; per-head columns to disk.
        rstd1 = np.empty(S)
        qkv_files = {}
        for j, name in enumerate("qkv"):
            for n in range(H):
                qkv_files[name, n] = np.lib.format.open_memmap(os.path.join(d, f"{name}{n}.npy"), mode="w+",
                                                               dtype=np.float64, shape=(S, dh))
        for rows in blocks:
            a, rstd1[rows] = rmsnorm(x[rows], w["g1"], EPS)
            for j, name in enumerate("qkv"):
                proj = a @ w["wqkv"][j * h:(j + 1) * h].T
                for n in range(H):
                    qkv_files[name, n][rows] = proj[:, n * dh:(n + 1) * dh]
        for m in qkv_files.values():
            m.flush()
        del qkv_files
        say("projections done")

        _per_head(_head_forward, d, H, workers)
        say("attention forward done")
        o = np.empty((S, h))
        for n in range(H):
            o[:, n * dh:(n + 1) * dh] = np.load(os.path.join(d, f"o{n}.npy"))

        # Out-projection + residual, RMSNorm2, MLP forward and backward, the
        # RMSNorm2 backward and the out-projection backward: all row-local.
        z = np.empty((S, h))
        dy = np.empty((S, h))
        dw1 = np.zeros((F, h))
        dw2 = np.zeros((h, F))
        dwo = np.zeros((h, h))
        dg2 = np.zeros(h)
        do_files = [np.lib.format.open_memmap(os.path.join(d, f"do{n}.npy"), mode="w+", dtype=np.float64,
                                              shape=(S, dh)) for n in range(H)]
        for rows in blocks:
            y = x[rows] + o[rows] @ w["wo"].T
            b, rstd2 = rmsnorm(y, w["g2"], EPS)
            u = b @ w["w1"].T
            g = gelu_tanh(u)
            z[rows] = y + g @ w["w2"].T
            dzb = dz[rows]
            dgl = dzb @ w["w2"]
            dw2 += dzb.T @ g
            du = dgl * gelu_tanh_grad(u)
            del g, u, dgl
            dw1 += du.T @ b
            db = du @ w["w1"]
            del du
            dyn, dg2b = rmsnorm_backward(db, y, rstd2, w["g2"])
            dg2 += dg2b
            dy[rows] = dzb + dyn
            dob = dy[rows] @ w["wo"]
            dwo += dy[rows].T @ o[rows]
            for n in range(H):
                do_files[n][rows] = dob[:, n * dh:(n + 1) * dh]
        for m in do_files:
            m.flush()
        del do_files
        say("MLP and out-projection done")

        _per_head(_head_backward, d, H, workers)
        say("attention backward done")

        # Projection backward and RMSNorm1 backward, per row block.
        grads = {name: [np.load(os.path.join(d, f"{name}{n}.npy"), mmap_mode="r") for n in range(H)]
                 for name in ("dq", "dk", "dv")}
        dx = np.empty((S, h))
        dwqkv = np.zeros((3 * h, h))
        dg1 = np.zeros(h)
        for rows in blocks:
            a, _ = rmsnorm(x[rows], w["g1"], EPS)
            dqkv = np.concatenate([np.concatenate([np.asarray(grads[name][n][rows]) for n in range(H)], axis=1)
                                   for name in ("dq", "dk", "dv")], axis=1)
            dwqkv += dqkv.T @ a
            da = dqkv @ w["wqkv"]
            dxn, dg1b = rmsnorm_backward(da, x[rows], rstd1[rows], w["g1"])
            dg1 += dg1b
            dx[rows] = dy[rows] + dxn
        del grads
        say("projection backward done")
        return dict(z=z, dx=dx, dg1=dg1, dwqkv=dwqkv, dwo=dwo, dg2=dg2, dw1=dw1, dw2=dw2)
    finally:
        if own:
            shutil.rmtree(d, ignore_errors=True)
