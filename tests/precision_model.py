"""CPU model of the CUDA path's rounding placement (test infrastructure).

It recomputes the layer in NumPy with fp32 accumulation and rounds, exactly
where the CUDA path stores a tensor-core operand, to that operand's type:

* placement "f16" (the CUDA path): a, Q, K, V, P, O, b, G and, in the
  backward, dU, dy, dO, P, dS and [dQ|dK|dV] are rounded to fp16 (RNE,
  subnormals included); P with the 2^7 factor the kernels give it, and the
  backward's gradients at the power-of-two scale 2^k the kernels take from
  max|dY| (largest |dY| 2^k in [8, 16)), so fp16's range limits are modelled
  too.  U (read only by GELU') is bf16, as on the GPU.
* placement "bf16": the same sites rounded to bf16 (the alternative the fp16
  placement replaced).

In both, the outputs z and dx are bf16, and the residual stream y, the
RMSNorm statistics, db, da and all weight gradients stay fp32, as on the GPU.
Weights and dY enter exactly (bf16 values; their fp16 copies are exact).
Comparing this model with the fp64 oracle measures the error floor of the
rounding placement, independent of how the kernels tile or order their sums.

It shares no code with the CUDA library and does not call it.
"""

from __future__ import annotations

import math

import numpy as np

from synth_inputs import bf16_bits, bits_to_f32


def rb(a) -> np.ndarray:
    """Round to bf16 (RNE) and widen back to float32."""
    return bits_to_f32(bf16_bits(np.asarray(a, dtype=np.float32)))


def rh(a, scale: float = 1.0) -> np.ndarray:
    """Round a * scale to fp16 (RNE, subnormals included), divide the scale
    back out, in float32."""
    a = np.asarray(a, dtype=np.float32)
    return (np.float32(scale) * a).astype(np.float16).astype(np.float32) / np.float32(scale)


def _gelu(u):
    return (0.5 * u * (1 + np.tanh(math.sqrt(2 / math.pi) * (u + 0.044715 * u ** 3)))).astype(np.float32)


def _gelu_grad(u):
    t = np.tanh(math.sqrt(2 / math.pi) * (u + 0.044715 * u ** 3))
    k = math.sqrt(2 / math.pi)
    return (0.5 * (1 + t) + 0.5 * u * (1 - t * t) * k * (1 + 3 * 0.044715 * u * u)).astype(np.float32)


def _rms(x, g):
    r = (1 / np.sqrt(np.mean(x.astype(np.float32) ** 2, axis=1) + 1e-5)).astype(np.float32)
    return (x * r[:, None] * g).astype(np.float32), r


def grad_scale(dY) -> float:
    """2^k with max|dY| * 2^k in [8, 16)."""
    m = float(np.max(np.abs(dY)))
    if m == 0.0:
        return 1.0
    _, E = math.frexp(m)
    return 2.0 ** (4 - E)


def layer(x, w, dY, H, placement="f16", block=512):
    """Forward and backward of the unsharded layer (global token order) with
    the rounding placement above.  x, dY: float32 [S, h] (bf16 values);
    w: float32 weights and gains.  Returns dict z, dx, dg1, dwqkv, dwo, dg2,
    dw1, dw2."""
    if placement == "f16":
        gs = grad_scale(dY)
        op = lambda t: rh(t)
        opP = lambda t: rh(t, 128.0)
        opg = lambda t: rh(t, gs)
    elif placement == "bf16":
        op = opP = opg = rb
    else:
        raise ValueError(placement)
    S, h = x.shape
    dh = h // H
    sc = 1.0 / math.sqrt(dh)
    Wq, Wk, Wv = w["wqkv"][:h], w["wqkv"][h:2 * h], w["wqkv"][2 * h:]
    a, r1 = _rms(x, w["g1"])
    ab = op(a)
    q, k, v = op(ab @ Wq.T), op(ab @ Wk.T), op(ab @ Wv.T)
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
            o[rows, c] = (opP(p) @ v[:kend, c]) / l[:, None]
            lse[n, rows] = m + np.log(l)
    ob = op(o)
    y = x + ob @ w["wo"].T
    b, r2 = _rms(y, w["g2"])
    bb = op(b)
    u = bb @ w["w1"].T
    G = op(_gelu(u))
    z = rb(y + G @ w["w2"].T)
    # backward
    dU = opg((dY @ w["w2"]) * _gelu_grad(rb(u)))
    dW2 = dY.T @ G
    dW1 = dU.T @ bb
    db = dU @ w["w1"]
    n2 = y * r2[:, None]
    dn = db * w["g2"]
    dy = dY + r2[:, None] * (dn - n2 * np.mean(dn * n2, 1, keepdims=True))
    dg2 = np.sum(db * n2, 0)
    dyb = opg(dy)
    dO = opg(dyb @ w["wo"])
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
            dv[:kend, c] += opP(p).T @ dO[rows, c]
            dp = dO[rows, c] @ v[:kend, c].T
            delta = np.sum(dO[rows, c] * ob[rows, c], 1)
            ds = opg(p * (dp - delta[:, None]))
            dq[rows, c] = (ds @ k[:kend, c]) * sc
            dk[:kend, c] += (ds.T @ q[rows, c]) * sc
    dqkv = opg(np.concatenate([dq, dk, dv], 1))
    dWqkv = dqkv.T @ ab
    da = dqkv @ w["wqkv"]
    n1 = x * r1[:, None]
    dn = da * w["g1"]
    dx = rb(dy + r1[:, None] * (dn - n1 * np.mean(dn * n1, 1, keepdims=True)))
    dg1 = np.sum(da * n1, 0)
    return dict(z=z, dx=dx, dg1=dg1, dwqkv=dWqkv, dwo=dWo, dg2=dg2, dw1=dW1, dw2=dW2)
