"""fp64 oracle of one folded Tensor-Sequence-Parallel (TSP) decoder layer.

TEST INFRASTRUCTURE ONLY: used by ``tests/``, ``__graft_entry__.smoke()`` and
the CPU legs of ``bench.py``; never by the library.  It shares no code with
the CUDA path.  Every computation is plain NumPy in float64 on inputs that the
caller has already rounded to bf16.

Sources (web pages on Zyphra's TSP; none prints an equation or a listing):

[Z1] "Zyphra TSP folds TP+SP onto one GPU axis, 2.6x throughput on 1,024
     MI300Xs" (zubnet.ai), paragraph 1: TP (weights) and SP (activations) are
     folded onto one device-mesh axis of size D; every device keeps 1/D of the
     model weights and 1/D of the sequence tokens.  Validated on a dense
     decoder-only 7B model (h=4096, 32 Q/KV heads, FFN x4, bf16), D=8.
[Z2] Same page, paragraph 2: for attention, the weight shards are broadcast
     one after another and each device applies them to its own tokens; then
     K/V are all-gathered, with a zigzag partition of the tokens for load
     balance.  For the MLP, a ring schedule rotates the weight shards by
     point-to-point steps, which removes the all-reduce that standard TP needs.
[Z4] Same page, paragraph 4: the MLP-without-all-reduce trick on its own.
[A1] "Zyphra TSP: 2.6x Faster AI Training Review" (ageofai.tools), "What's
     New": the folded axis cuts both parameter and activation memory.

What the pages leave open is read as follows (each reading is listed with its
reason in the design notes):

* 2D zigzag chunks of c = S/(2D) tokens; rank r owns chunk r and chunk
  2D-1-r, in ascending token order.
* Attention shard t = heads [t*H/D, (t+1)*H/D): rows of Wq/Wk/Wv, columns of
  Wo.  MLP shard s = FFN units [s*F/D, (s+1)*F/D): rows of W1, columns of W2.
* Broadcast step t sends shard t; the out-projection partial sums follow the
  same cycle, t = 0..D-1.
* Ring: rank r starts with its own MLP shard and, after each step, receives
  the shard held by rank r+1 (mod D); so at step t it holds shard (r+t) mod D.
* Layer: pre-RMSNorm (eps 1e-5 inside the square root, gains g1, g2), causal
  softmax attention with scale 1/sqrt(dh) and key <= query, no positional
  encoding, no bias, GELU with the tanh approximation, two residuals.
* Backward: the exact gradient; weight-gradient pieces are summed at the
  shard's owner in rank order 0..D-1; key/value gradients are summed at the
  key's owner (reduce-scatter) in rank order.

Parity pins for every function live in ``tests/test_oracle_pins.py``.
"""

from __future__ import annotations

import math

import numpy as np

EPS = 1e-5
_GELU_K = math.sqrt(2.0 / math.pi)
_GELU_A = 0.044715
_ROW_BLOCK = 256


# ---------------------------------------------------------------------------
# Partition and schedules  [Z1], [Z2]
# ---------------------------------------------------------------------------

def zigzag_map(S: int, D: int) -> np.ndarray:
    """Zigzag token partition [Z2].

    The sequence is cut into 2D chunks of c = S/(2D) tokens; rank r holds chunk
    r followed by chunk 2D-1-r.  Returns ``m`` of shape [D, L] (L = S/D) with
    ``m[r, i]`` = the global position of rank r's i-th token."""
    if S % (2 * D):
        raise ValueError("S must be a multiple of 2D")
    c = S // (2 * D)
    m = np.empty((D, S // D), dtype=np.int64)
    for r in range(D):
        m[r, :c] = np.arange(r * c, (r + 1) * c)
        m[r, c:] = np.arange((2 * D - 1 - r) * c, (2 * D - r) * c)
    return m


def causal_pairs_per_rank(zig: np.ndarray) -> np.ndarray:
    """Number of (query, key) pairs with key <= query that each rank's queries
    attend to, counted by comparing every key position with every query
    position (brute force)."""
    D, L = zig.shape
    S = D * L
    keys = np.arange(S)
    out = np.zeros(D, dtype=np.int64)
    for r in range(D):
        for i0 in range(0, L, 512):
            q = zig[r, i0:i0 + 512]
            out[r] += int(np.count_nonzero(keys[None, :] <= q[:, None]))
    return out


def shard_schedule(D: int, phase: int) -> np.ndarray:
    """Which weight shard every rank applies at every step, ``sched[t, r]``.

    phase 0, attention broadcast [Z2]: at step t rank t broadcasts its shard and
    every rank applies it, so ``sched[t, r] = t``.
    phase 1, MLP ring [Z2]: rank r starts with shard r; after each step it
    receives what rank r+1 (mod D) held.  The ring is simulated hop by hop."""
    sched = np.empty((D, D), dtype=np.int64)
    if phase == 0:
        for t in range(D):
            sched[t, :] = t
        return sched
    if phase != 1:
        raise ValueError("phase must be 0 (broadcast) or 1 (ring)")
    held = list(range(D))
    for t in range(D):
        sched[t, :] = held
        held = [held[(r + 1) % D] for r in range(D)]
    return sched


def head_cols(t: int, H: int, D: int, dh: int) -> slice:
    """Feature columns of attention shard t: heads [t*H/D, (t+1)*H/D)."""
    hp = H // D
    return slice(t * hp * dh, (t + 1) * hp * dh)


def ffn_units(s: int, F: int, D: int) -> slice:
    """FFN units of MLP shard s: [s*F/D, (s+1)*F/D)."""
    fp = F // D
    return slice(s * fp, (s + 1) * fp)


# ---------------------------------------------------------------------------
# Token-local pieces of the layer (workload specification)
# ---------------------------------------------------------------------------

def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float = EPS):
    """RMSNorm (Zhang & Sennrich 2019): x / sqrt(mean(x^2) + eps) * g, per row.
    Returns (output, rstd) with rstd of shape [rows]."""
    rstd = 1.0 / np.sqrt(np.mean(x * x, axis=-1) + eps)
    return x * rstd[:, None] * g[None, :], rstd


def rmsnorm_backward(dout: np.ndarray, x: np.ndarray, rstd: np.ndarray, g: np.ndarray):
    """Gradient of ``rmsnorm`` w.r.t. its input and its gain.

    With n = x*rstd and out = n*g: dn = dout*g,
    dx = rstd * (dn - n * mean(dn*n)), dg = sum over rows of dout*n."""
    n = x * rstd[:, None]
    dn = dout * g[None, :]
    dx = rstd[:, None] * (dn - n * np.mean(dn * n, axis=-1, keepdims=True))
    dg = np.sum(dout * n, axis=0)
    return dx, dg


def gelu_tanh(u: np.ndarray) -> np.ndarray:
    """GELU, tanh approximation (Hendrycks & Gimpel 2016):
    0.5 u (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3)))."""
    return 0.5 * u * (1.0 + np.tanh(_GELU_K * (u + _GELU_A * u ** 3)))


def gelu_tanh_grad(u: np.ndarray) -> np.ndarray:
    """d/du of ``gelu_tanh``."""
    t = np.tanh(_GELU_K * (u + _GELU_A * u ** 3))
    return 0.5 * (1.0 + t) + 0.5 * u * (1.0 - t * t) * _GELU_K * (1.0 + 3.0 * _GELU_A * u * u)


# ---------------------------------------------------------------------------
# Causal softmax attention (decoder-only layer [Z1])
# ---------------------------------------------------------------------------

def causal_attention(q, k, v, qpos, H):
    """Softmax attention of queries at global positions ``qpos`` against keys
    and values stored at global positions 0..Sk-1; key k is visible to a query
    at position p iff k <= p; scale 1/sqrt(dh).

    Every query row is independent; rows are taken ``_ROW_BLOCK`` at a time
    only to bound memory, and keys past the block's last position (all masked)
    are not formed.  Returns O [Lq, h] and the natural-log logsumexp
    LSE [H, Lq] of the scaled scores."""
    Lq, h = q.shape
    dh = h // H
    scale = 1.0 / math.sqrt(dh)
    o = np.zeros((Lq, h))
    lse = np.zeros((H, Lq))
    kpos = np.arange(k.shape[0])
    for i0 in range(0, Lq, _ROW_BLOCK):
        rows = slice(i0, min(i0 + _ROW_BLOCK, Lq))
        qp = qpos[rows]
        kend = int(qp.max()) + 1
        masked = kpos[None, :kend] > qp[:, None]
        for n in range(H):
            c = slice(n * dh, (n + 1) * dh)
            s = (q[rows, c] @ k[:kend, c].T) * scale
            s[masked] = -np.inf
            m = s.max(axis=1)
            p = np.exp(s - m[:, None])
            l = p.sum(axis=1)
            o[rows, c] = (p @ v[:kend, c]) / l[:, None]
            lse[n, rows] = m + np.log(l)
    return o, lse


def causal_attention_backward(q, k, v, o, do, lse, qpos, H):
    """Gradient of ``causal_attention`` for upstream dO.

    P = exp(s - LSE); dV = P^T dO; dP = dO V^T; Delta = rowsum(dO * O);
    dS = P * (dP - Delta); dQ = dS K / sqrt(dh); dK = dS^T Q / sqrt(dh).
    Returns dQ [Lq, h] and dK, dV [Sk, h] (key-side gradients at global rows)."""
    Lq, h = q.shape
    dh = h // H
    scale = 1.0 / math.sqrt(dh)
    dq = np.zeros((Lq, h))
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    kpos = np.arange(k.shape[0])
    for i0 in range(0, Lq, _ROW_BLOCK):
        rows = slice(i0, min(i0 + _ROW_BLOCK, Lq))
        qp = qpos[rows]
        kend = int(qp.max()) + 1
        masked = kpos[None, :kend] > qp[:, None]
        for n in range(H):
            c = slice(n * dh, (n + 1) * dh)
            s = (q[rows, c] @ k[:kend, c].T) * scale
            p = np.exp(s - lse[n, rows][:, None])
            p[masked] = 0.0
            dv[:kend, c] += p.T @ do[rows, c]
            dp = do[rows, c] @ v[:kend, c].T
            delta = np.sum(do[rows, c] * o[rows, c], axis=1)
            ds = p * (dp - delta[:, None])
            dq[rows, c] = (ds @ k[:kend, c]) * scale
            dk[:kend, c] += (ds.T @ q[rows, c]) * scale
    return dq, dk, dv


# ---------------------------------------------------------------------------
# The unsharded layer (D = 1): the result that folding must not change [Z1]
# ---------------------------------------------------------------------------

def _as64(w):
    return {k: np.asarray(v, dtype=np.float64) for k, v in w.items()}


def layer_forward(x, w, H, eps=EPS):
    """Unsharded pre-RMSNorm decoder layer on tokens in global order.
    ``w`` holds wqkv [3h,h], wo [h,h], w1 [F,h], w2 [h,F], g1 [h], g2 [h].
    Returns (z, cache)."""
    w = _as64(w)
    x = np.asarray(x, dtype=np.float64)
    S, h = x.shape
    a, rstd1 = rmsnorm(x, w["g1"], eps)
    q = a @ w["wqkv"][:h].T
    k = a @ w["wqkv"][h:2 * h].T
    v = a @ w["wqkv"][2 * h:].T
    o, lse = causal_attention(q, k, v, np.arange(S), H)
    y = x + o @ w["wo"].T
    b, rstd2 = rmsnorm(y, w["g2"], eps)
    u = b @ w["w1"].T
    z = y + gelu_tanh(u) @ w["w2"].T
    cache = dict(x=x, a=a, rstd1=rstd1, q=q, k=k, v=v, o=o, lse=lse, y=y, b=b, rstd2=rstd2, u=u)
    return z, cache


def layer_backward(dz, w, H, cache):
    """Exact gradient of ``layer_forward`` for upstream dz (global order)."""
    w = _as64(w)
    dz = np.asarray(dz, dtype=np.float64)
    c = cache
    h = c["x"].shape[1]
    S = c["x"].shape[0]
    g = gelu_tanh(c["u"])
    dg = dz @ w["w2"]
    dw2 = dz.T @ g
    du = dg * gelu_tanh_grad(c["u"])
    dw1 = du.T @ c["b"]
    db = du @ w["w1"]
    dyn, dg2 = rmsnorm_backward(db, c["y"], c["rstd2"], w["g2"])
    dy = dz + dyn
    do = dy @ w["wo"]
    dwo = dy.T @ c["o"]
    dq, dk, dv = causal_attention_backward(c["q"], c["k"], c["v"], c["o"], do, c["lse"], np.arange(S), H)
    dqkv = np.concatenate([dq, dk, dv], axis=1)
    dwqkv = dqkv.T @ c["a"]
    da = dqkv @ w["wqkv"]
    dxn, dg1 = rmsnorm_backward(da, c["x"], c["rstd1"], w["g1"])
    dx = dy + dxn
    return dict(dx=dx, dg1=dg1, dwqkv=dwqkv, dwo=dwo, dg2=dg2, dw1=dw1, dw2=dw2)


# ---------------------------------------------------------------------------
# The folded layer, simulated rank by rank  [Z1], [Z2], [Z4]
# ---------------------------------------------------------------------------

def _split_ranks(a, D):
    L = a.shape[0] // D
    return [a[r * L:(r + 1) * L] for r in range(D)]


def tsp_layer_forward(x_local, w, H, D, eps=EPS):
    """Forward of the folded layer over D simulated ranks.

    ``x_local`` is [S, h] in rank-major zigzag order (rank 0's L tokens, then
    rank 1's, ...).  Each step is done per rank with explicit messages:
    the broadcast of attention shards, the all-gather of K/V into global
    order, and the ring of MLP shards whose partial sums stay on the rank.
    Returns (z_local [S, h] rank-major, cache)."""
    w = _as64(w)
    x_local = np.asarray(x_local, dtype=np.float64)
    S, h = x_local.shape
    L = S // D
    F = w["w1"].shape[0]
    dh = h // H
    zig = zigzag_map(S, D)
    xr = _split_ranks(x_local, D)

    # RMSNorm1 is token-local.
    a, rstd1 = [], []
    for r in range(D):
        ar, sr = rmsnorm(xr[r], w["g1"], eps)
        a.append(ar)
        rstd1.append(sr)

    # Attention projections under the broadcast schedule [Z2]: at step t the
    # owner of shard t sends its Wq/Wk/Wv rows and every rank applies them to
    # its own tokens.
    bcast = shard_schedule(D, 0)
    Q = [np.zeros((L, h)) for _ in range(D)]
    K = [np.zeros((L, h)) for _ in range(D)]
    V = [np.zeros((L, h)) for _ in range(D)]
    for t in range(D):
        for r in range(D):
            sh = int(bcast[t, r])
            cols = head_cols(sh, H, D, dh)
            msg_q = w["wqkv"][0 * h:1 * h][cols]
            msg_k = w["wqkv"][1 * h:2 * h][cols]
            msg_v = w["wqkv"][2 * h:3 * h][cols]
            Q[r][:, cols] = a[r] @ msg_q.T
            K[r][:, cols] = a[r] @ msg_k.T
            V[r][:, cols] = a[r] @ msg_v.T

    # All-gather of K/V [Z2]: every rank's rows land at their global positions.
    Kg = np.zeros((S, h))
    Vg = np.zeros((S, h))
    for r in range(D):
        Kg[zig[r]] = K[r]
        Vg[zig[r]] = V[r]
    del K, V

    # Causal attention of each rank's local queries against the gathered K/V.
    O, lse = [], []
    for r in range(D):
        o_r, l_r = causal_attention(Q[r], Kg, Vg, zig[r], H)
        O.append(o_r)
        lse.append(l_r)

    # Out-projection: the same broadcast cycle; partial sums over head groups
    # are added in step order t = 0..D-1, then the residual.
    y, b, rstd2 = [], [], []
    for r in range(D):
        acc = np.zeros((L, h))
        for t in range(D):
            cols = head_cols(int(bcast[t, r]), H, D, dh)
            acc += O[r][:, cols] @ w["wo"][:, cols].T
        yr = xr[r] + acc
        br, sr = rmsnorm(yr, w["g2"], eps)
        y.append(yr)
        b.append(br)
        rstd2.append(sr)

    # MLP ring [Z2], [Z4]: at step t rank r holds FFN shard (r+t) mod D; its
    # partial sum of GELU(b W1_s^T) W2_s^T stays in the rank's own
    # accumulator, so no all-reduce ever combines ranks.
    ring = shard_schedule(D, 1)
    U = [np.zeros((L, F)) for _ in range(D)]
    z = []
    accs = [np.zeros((L, h)) for _ in range(D)]
    for t in range(D):
        for r in range(D):
            units = ffn_units(int(ring[t, r]), F, D)
            u = b[r] @ w["w1"][units].T
            U[r][:, units] = u
            accs[r] += gelu_tanh(u) @ w["w2"][:, units].T
    for r in range(D):
        z.append(y[r] + accs[r])

    cache = dict(zig=zig, x=xr, a=a, rstd1=rstd1, Q=Q, Kg=Kg, Vg=Vg, O=O, lse=lse,
                 y=y, b=b, rstd2=rstd2, U=U, H=H, D=D)
    return np.concatenate(z, axis=0), cache


def tsp_ring_mlp(b_local, w1, w2, resid_local, D):
    """[Z2], [Z4]: the MLP in its ring schedule on its own.  b_local and
    resid_local are rank-major [S][h] (rank r holds rows r*L .. (r+1)*L - 1);
    at step t rank r applies FFN shard (r+t) mod D to its own rows, and the
    partial sums stay in that rank's accumulator, which is added to the
    residual at the end (no sum across ranks)."""
    b_local = np.asarray(b_local, dtype=np.float64)
    S, h = b_local.shape
    F = w1.shape[0]
    L = S // D
    ring = shard_schedule(D, 1)
    accs = [np.zeros((L, h)) for _ in range(D)]
    for t in range(D):
        for r in range(D):
            units = ffn_units(int(ring[t, r]), F, D)
            accs[r] += gelu_tanh(b_local[r * L:(r + 1) * L] @ w1[units].T) @ w2[:, units].T
    return np.asarray(resid_local, dtype=np.float64) + np.concatenate(accs, axis=0)


def tsp_layer_backward(dz_local, w, cache):
    """Exact gradient of ``tsp_layer_forward``, rank by rank.

    Token-local gradients stay on their rank.  Each weight shard's gradient is
    the sum of the ranks' pieces, added at the shard's owner in rank order
    0..D-1.  Key/value gradients, formed at global rows by every rank's queries,
    are summed (rank order) and handed back to the key's owner: the reverse of
    the all-gather.  Returns dx (rank-major), dg1, dwqkv, dwo, dg2, dw1, dw2."""
    w = _as64(w)
    c = cache
    H, D = c["H"], c["D"]
    zig = c["zig"]
    dz = _split_ranks(np.asarray(dz_local, dtype=np.float64), D)
    L, h = dz[0].shape
    F = w["w1"].shape[0]
    dh = h // H
    S = L * D
    bcast = shard_schedule(D, 0)
    ring = shard_schedule(D, 1)

    # Ring MLP backward: the shards travel the ring again.
    piece_w1 = [[None] * D for _ in range(D)]
    piece_w2 = [[None] * D for _ in range(D)]
    db = [np.zeros((L, h)) for _ in range(D)]
    for t in range(D):
        for r in range(D):
            s = int(ring[t, r])
            units = ffn_units(s, F, D)
            u = c["U"][r][:, units]
            dgl = dz[r] @ w["w2"][:, units]
            du = dgl * gelu_tanh_grad(u)
            piece_w2[s][r] = dz[r].T @ gelu_tanh(u)
            piece_w1[s][r] = du.T @ c["b"][r]
            db[r] += du @ w["w1"][units]
    dw1 = np.zeros((F, h))
    dw2 = np.zeros((h, F))
    for s in range(D):
        units = ffn_units(s, F, D)
        for r in range(D):
            dw2[:, units] += piece_w2[s][r]
            dw1[units] += piece_w1[s][r]

    # RMSNorm2 backward plus the residual.
    dy = []
    dg2 = np.zeros(h)
    for r in range(D):
        dyn, dgr = rmsnorm_backward(db[r], c["y"][r], c["rstd2"][r], w["g2"])
        dy.append(dz[r] + dyn)
        dg2 += dgr

    # Out-projection backward, broadcast cycle.
    dO = [np.zeros((L, h)) for _ in range(D)]
    dwo = np.zeros((h, h))
    for t in range(D):
        pieces = []
        for r in range(D):
            cols = head_cols(int(bcast[t, r]), H, D, dh)
            dO[r][:, cols] = dy[r] @ w["wo"][:, cols]
            pieces.append(dy[r].T @ c["O"][r][:, cols])
        cols = head_cols(t, H, D, dh)
        for r in range(D):
            dwo[:, cols] += pieces[r]

    # Attention backward; key-side gradients are reduced to the keys' owners.
    dQ = []
    dKg = np.zeros((S, h))
    dVg = np.zeros((S, h))
    for r in range(D):
        dq, dk, dv = causal_attention_backward(c["Q"][r], c["Kg"], c["Vg"], c["O"][r], dO[r],
                                               c["lse"][r], zig[r], H)
        dQ.append(dq)
        dKg += dk
        dVg += dv
    dK = [dKg[zig[r]] for r in range(D)]
    dV = [dVg[zig[r]] for r in range(D)]

    # Projection backward, broadcast cycle.
    da = [np.zeros((L, h)) for _ in range(D)]
    dwqkv = np.zeros((3 * h, h))
    for t in range(D):
        cols = head_cols(t, H, D, dh)
        for r in range(D):
            for j, g in enumerate((dQ[r], dK[r], dV[r])):
                wsh = w["wqkv"][j * h:(j + 1) * h][cols]
                da[r] += g[:, cols] @ wsh
                dwqkv[j * h:(j + 1) * h][cols] += g[:, cols].T @ c["a"][r]

    # RMSNorm1 backward plus the residual.
    dx = []
    dg1 = np.zeros(h)
    for r in range(D):
        dxn, dgr = rmsnorm_backward(da[r], c["x"][r], c["rstd1"][r], w["g1"])
        dx.append(dy[r] + dxn)
        dg1 += dgr
    return dict(dx=np.concatenate(dx, axis=0), dg1=dg1, dwqkv=dwqkv, dwo=dwo, dg2=dg2,
                dw1=dw1, dw2=dw2)


# ---------------------------------------------------------------------------
# A stack of folded layers  [Z1]: the measured model is a stack of these
# layers (a 7B decoder); between layers the tensors are bf16 (the layer's
# boundary dtype)
# ---------------------------------------------------------------------------

def round_bf16(x):
    """Round fp64 values to the nearest bfloat16 value (8 significand bits,
    ties to even), returned as fp64.  The values here are finite and far from
    bfloat16's range limits."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                    # x = m 2^e with 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def tsp_stack_forward(x_local, ws, H, D, round_interfaces=True):
    """z = layer_{L-1}(... layer_0(x)) with every layer the folded layer of
    ``tsp_layer_forward`` (weights ``ws[i]`` for layer i); the activation
    between two layers is rounded to bf16 unless ``round_interfaces`` is
    False.  Returns (z, caches), z unrounded."""
    caches = []
    cur = np.asarray(x_local, dtype=np.float64)
    z = None
    for i, w in enumerate(ws):
        z, cache = tsp_layer_forward(cur, w, H, D)
        caches.append(cache)
        cur = round_bf16(z) if round_interfaces and i < len(ws) - 1 else z
    return z, caches


def tsp_stack_backward(dz_local, ws, caches, round_interfaces=True):
    """Gradients of the stack: layer i's backward (``tsp_layer_backward``) on
    the gradient of its output, from the last layer down; the gradient
    passed to the layer below is rounded to bf16 unless ``round_interfaces``
    is False.  Returns one gradient dict per layer; the stack's dx is
    grads[0]["dx"]."""
    grads = [None] * len(ws)
    g = np.asarray(dz_local, dtype=np.float64)
    for i in reversed(range(len(ws))):
        grads[i] = tsp_layer_backward(g, ws[i], caches[i])
        g = round_bf16(grads[i]["dx"]) if round_interfaces and i > 0 else grads[i]["dx"]
    return grads


def tsp_forward_rows(x_local, w, H, D, rows, eps=EPS):
    """Folded forward restricted to the rank-major rows ``rows``.

    K and V are formed for all S tokens (broadcast schedule, then all-gather),
    because every query may see any earlier key; everything else is
    token-local and is evaluated for the requested rows only, with the same
    step order and partial-sum order as ``tsp_layer_forward``.
    Returns z for those rows, [len(rows), h]."""
    w = _as64(w)
    S, h = x_local.shape
    L = S // D
    F = w["w1"].shape[0]
    dh = h // H
    zig = zigzag_map(S, D)
    bcast = shard_schedule(D, 0)
    ring = shard_schedule(D, 1)
    rows = np.asarray(rows, dtype=np.int64)

    Kg = np.zeros((S, h))
    Vg = np.zeros((S, h))
    for r in range(D):
        a_r, _ = rmsnorm(np.asarray(x_local[r * L:(r + 1) * L], dtype=np.float64), w["g1"], eps)
        for t in range(D):
            cols = head_cols(int(bcast[t, r]), H, D, dh)
            Kg[zig[r], cols] = a_r @ w["wqkv"][h:2 * h][cols].T
            Vg[zig[r], cols] = a_r @ w["wqkv"][2 * h:][cols].T
        del a_r

    out = np.zeros((len(rows), h))
    for r in range(D):
        sel = np.nonzero((rows >= r * L) & (rows < (r + 1) * L))[0]
        if len(sel) == 0:
            continue
        xl = np.asarray(x_local[rows[sel]], dtype=np.float64)
        a_r, _ = rmsnorm(xl, w["g1"], eps)
        q = np.zeros((len(sel), h))
        for t in range(D):
            cols = head_cols(int(bcast[t, r]), H, D, dh)
            q[:, cols] = a_r @ w["wqkv"][:h][cols].T
        qpos = zig[r][rows[sel] - r * L]
        o, _ = causal_attention(q, Kg, Vg, qpos, H)
        acc = np.zeros((len(sel), h))
        for t in range(D):
            cols = head_cols(int(bcast[t, r]), H, D, dh)
            acc += o[:, cols] @ w["wo"][:, cols].T
        y = xl + acc
        b, _ = rmsnorm(y, w["g2"], eps)
        acc = np.zeros((len(sel), h))
        for t in range(D):
            units = ffn_units(int(ring[t, r]), F, D)
            acc += gelu_tanh(b @ w["w1"][units].T) @ w["w2"][:, units].T
        out[sel] = y + acc
    return out
