"""CPU model of the CUDA path's rounding placement (test infrastructure).

It recomputes the layer in NumPy with fp32 accumulation and rounds to bf16
(round-to-nearest-even) exactly the tensors that the CUDA path stores as bf16
operands of a contraction: a, Q, K, V, P, O, b, G, U (for GELU'), dU, dy, dO,
P and dS inside the attention backward, [dQ|dK|dV], and the bf16 outputs z and
dx.  The residual stream y, the RMSNorm statistics, db, da and all weight
gradients stay fp32, as on the GPU.  Comparing this model with the fp64 oracle
measures the error floor that any arithmetic with this rounding placement has,
independent of how the kernels tile or order their sums.

It shares no code with the CUDA library and does not call it.
"""

from __future__ import annotations

import math

import numpy as np

from synth_inputs import bf16_bits, bits_to_f32


def rb(a) -> np.ndarray:
    """Round to bf16 (RNE) and widen back to float32."""
    return bits_to_f32(bf16_bits(np.asarray(a, dtype=np.float32)))


def _gelu(u):
    return (0.5 * u * (1 + np.tanh(math.sqrt(2 / math.pi) * (u + 0.044715 * u ** 3)))).astype(np.float32)


def _gelu_grad(u):
    t = np.tanh(math.sqrt(2 / math.pi) * (u + 0.044715 * u ** 3))
    k = math.sqrt(2 / math.pi)
    return (0.5 * (1 + t) + 0.5 * u * (1 - t * t) * k * (1 + 3 * 0.044715 * u * u)).astype(np.float32)


def _rms(x, g):
    r = (1 / np.sqrt(np.mean(x.astype(np.float32) ** 2, axis=1) + 1e-5)).astype(np.float32)
    return (x * r[:, None] * g).astype(np.float32), r


def bf16_layer(x, w, dY, H, block=512):
    """Forward and backward of the unsharded layer (global token order) with
    the rounding placement above.  x, dY: float32 [S, h] (bf16 values);
    w: float32 weights and gains.  Returns dict z, dx, dg1, dwqkv, dwo, dg2,
    dw1, dw2."""
    S, h = x.shape
    dh = h // H
    sc = 1.0 / math.sqrt(dh)
    Wq, Wk, Wv = w["wqkv"][:h], w["wqkv"][h:2 * h], w["wqkv"][2 * h:]
    a, r1 = _rms(x, w["g1"])
    ab = rb(a)
    q, k, v = rb(ab @ Wq.T), rb(ab @ Wk.T), rb(ab @ Wv.T)
    o = np.zeros((S, h), np.float32)
    lse = np.zeros((H, S), np.float32)
    for i0 in range(0, S, block):
        rows = slice(i0, min(i0 + block, S))
        kend = rows.stop
        mask = np.arange(kend)[None, :] > np.arange(i0, kend)[:, None]
        for n in range(H):
            c = slice(n * dh, (n + 1) * dh)
            s = (q[rows, c] @ k[:kend, c].T) * sc
            s[mask] = -np.inf
            m = s.max(1)
            p = np.exp(s - m[:, None])
            l = p.sum(1)
            o[rows, c] = (rb(p) @ v[:kend, c]) / l[:, None]
            lse[n, rows] = m + np.log(l)
    ob = rb(o)
    y = x + ob @ w["wo"].T
    b, r2 = _rms(y, w["g2"])
    bb = rb(b)
    u = bb @ w["w1"].T
    G = rb(_gelu(u))
    z = rb(y + G @ w["w2"].T)
    # backward
    dU = rb((dY @ w["w2"]) * _gelu_grad(rb(u)))
    dW2 = dY.T @ G
    dW1 = dU.T @ bb
    db = dU @ w["w1"]
    n2 = y * r2[:, None]
    dn = db * w["g2"]
    dy = dY + r2[:, None] * (dn - n2 * np.mean(dn * n2, 1, keepdims=True))
    dg2 = np.sum(db * n2, 0)
    dyb = rb(dy)
    dO = rb(dyb @ w["wo"])
    dWo = dyb.T @ ob
    dq = np.zeros((S, h), np.float32)
    dk = np.zeros_like(dq)
    dv = np.zeros_like(dq)
    for i0 in range(0, S, block):
        rows = slice(i0, min(i0 + block, S))
        kend = rows.stop
        mask = np.arange(kend)[None, :] > np.arange(i0, kend)[:, None]
        for n in range(H):
            c = slice(n * dh, (n + 1) * dh)
            s = (q[rows, c] @ k[:kend, c].T) * sc
            p = np.exp(s - lse[n, rows][:, None])
            p[mask] = 0
            dv[:kend, c] += rb(p).T @ dO[rows, c]
            dp = dO[rows, c] @ v[:kend, c].T
            delta = np.sum(dO[rows, c] * ob[rows, c], 1)
            ds = rb(p * (dp - delta[:, None]))
            dq[rows, c] = (ds @ k[:kend, c]) * sc
            dk[:kend, c] += (ds.T @ q[rows, c]) * sc
    dqkv = rb(np.concatenate([dq, dk, dv], 1))
    dWqkv = dqkv.T @ ab
    da = dqkv @ w["wqkv"]
    n1 = x * r1[:, None]
    dn = da * w["g1"]
    dx = rb(dy + r1[:, None] * (dn - n1 * np.mean(dn * n1, 1, keepdims=True)))
    dg1 = np.sum(da * n1, 0)
    return dict(z=z, dx=dx, dg1=dg1, dwqkv=dWqkv, dwo=dWo, dg2=dg2, dw1=dW1, dw2=dW2)
