"""CPU oracle for the HSTU layer: TEST INFRASTRUCTURE, never part of the product path.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline / reference
leg) may import or run anything in this directory. The CUDA library never calls it and shares
no code, table or constant generator with it.

Plain numpy, float64 throughout, written to be checked against the pages by eye. Library
primitives used as single steps: matrix product, sort/searchsorted, ``np.add.at``. Rows are
evaluated independently where a function accepts ``rows`` (each output row of the attention is
defined on its own, so computing a subset of rows is the same definition, not a reordering).

Pages followed (cited by title and section):

* "4.4 Scaling Recommendation Models" (LLM learning path, part 4), section "Generative
  Recommenders and HSTU": the three layer equations U,V,Q,K = Split(phi1(f1(X))),
  AV = phi2(QK^T + rab^{p,t})V, Y = f2(Norm(AV) (.) U); the "Pointwise aggregated attention"
  bullet (SiLU instead of softmax, constant normaliser such as the sequence length); the
  "Efficiency tricks" paragraph (variable-length kernels, stochastic length, M-FALCON).
  Section "Code": the HSTU sketch (chunk order u, v, q, k; per-head view; causal lower
  triangle including the diagonal; division by n; LayerNorm of AV over the full model width;
  residual added after f2).
* "HSTU: The First Exploration of the Scaling Law" (fun-rec 7.1), section 7.1.4
  "Innovation 1" (pointwise aggregation with SiLU), "Innovation 2" (bias from position and
  time differences), "Innovation 3" (Norm(AV) (.) U gating); section 7.1.5 "Stochastic
  Length" and "M-FALCON" (candidates see the cached history, not each other).

Readings where the pages are silent, garbled or disagree:

R1  No input LayerNorm before f1 (the equations have none); the sketch's extra one is the
    variant ``layer_fwd_norm_in`` (f1 reads LayerNorm_in(X), the residual adds X).
R2  N is a constant runtime scalar (``inv_N`` = 1/N), never the per-batch maximum length.
R3  The causal mask keeps j <= i (diagonal included), as in the sketch.
R4  rab_pos and rab_time are shared by all heads.
R5  time bucket = min(n_buckets-1, floor(ln(max(t_i - t_j, 1)) / 0.301)), evaluated exactly:
    bucket(v) = #{k in 1..n_buckets-1 : tau_k <= v}, tau_k = ceil(exp(0.301 k)) computed with
    60-digit decimal arithmetic (exp(0.301 k) is never an integer for k >= 1).
R6  rab_pos is indexed by clip(i - j, -(L-1), L-1) + L - 1 with L = pos_max_len
    (table of 2L-1 entries); a pair further apart than L-1 uses the last entry.
R7  AV is a matrix product (the fun-rec formula's elementwise product is a typo; the first
    page's equation and sketch multiply by V).
R8  Block wiring follows the first page: no output LayerNorm, residual added after f2.
R9  f1 and f2 carry biases; the LayerNorm is affine (gamma, beta), eps = 1e-5, biased
    variance, normalising over all d_model features of a token.
R10 Stochastic Length keeps L = min(n, floor(n**(alpha/2) + 1/2)) tokens, the L tokens with the
    smallest random keys (ties by position), in their original order; timestamps travel with
    the kept tokens and positions are renumbered 0..L-1.
R11 M-FALCON: a candidate attends to every token of its user's prefix and to itself; it sits at
    position n (the prefix length) with the request timestamp, so its result equals the last
    row of a causal forward over prefix + [candidate].
R12 The richer bias f(p_i - p_j, t_i - t_j, type_i, type_j) of "HSTU: The First Exploration of
    the Scaling Law", 7.1.4 Innovation 2, whose form the page does not give, is read as the sum of
    three looked-up terms: rab_pos[idx(p_i - p_j)] + rab_time[bucket(t_i - t_j)] +
    rab_type[type_i, type_j], each table either shared by the heads or with one slice per head
    (the first page's sketch keeps a per-head bias table). Token types are small integers.

Parity pins for every function live in ``tests/test_oracle_pins.py``; none is unpinned.
"""
from __future__ import annotations

import decimal
from typing import List, Optional, Sequence

import numpy as np

LN_EPS = 1e-5
BUCKET_WIDTH = "0.301"


# ----------------------------------------------------------------------------------------------
# Elementwise nonlinearity (phi1 = phi2 = SiLU)
# ----------------------------------------------------------------------------------------------

def silu(z: np.ndarray) -> np.ndarray:
    """SiLU(z) = z * sigmoid(z) ("4.4 Scaling Recommendation Models", HSTU layer: phi1, phi2)."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def silu_grad(z: np.ndarray) -> np.ndarray:
    """d SiLU / dz = sigmoid(z) * (1 + z * (1 - sigmoid(z)))."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        sg = 1.0 / (1.0 + np.exp(-z))
    return sg * (1.0 + z * (1.0 - sg))


# ----------------------------------------------------------------------------------------------
# Relative attention bias indices (rab^{p,t})
# ----------------------------------------------------------------------------------------------

def time_bucket_thresholds(n_buckets: int = 128, width: str = BUCKET_WIDTH) -> np.ndarray:
    """tau_k = ceil(exp(width * k)) for k = 1..n_buckets-1, exact (reading R5).

    "HSTU: The First Exploration of the Scaling Law", 7.1.4 Innovation 2: the bias depends on
    the time difference t_i - t_j; the bucketing ln(max(dt,1)) / 0.301 is the workload's
    stated scheme.
    """
    ctx = decimal.Context(prec=60, rounding=decimal.ROUND_HALF_EVEN)
    w = decimal.Decimal(width)
    taus = []
    for k in range(1, n_buckets):
        e = ctx.exp(w * k)
        taus.append(int(e.to_integral_value(rounding=decimal.ROUND_CEILING)))
    assert taus[-1] < 2 ** 63
    return np.array(taus, dtype=np.int64)


def time_bucket(dt, thresholds: np.ndarray) -> np.ndarray:
    """bucket(dt) = #{k : tau_k <= max(dt, 1)} = min(n_buckets-1, floor(ln(max(dt,1))/width))."""
    v = np.maximum(np.asarray(dt, dtype=np.int64), 1)
    return np.searchsorted(thresholds, v, side="right").astype(np.int64)


def time_diff(ts_q, ts_k) -> np.ndarray:
    """All differences t_q - t_k ([len(ts_q), len(ts_k)], int64), exact for any int64 inputs.

    The bias depends on the true difference of two timestamps ("HSTU: The First Exploration of the
    Scaling Law", 7.1.4 Innovation 2). When two int64 timestamps are more than 2^63 apart their
    difference has no int64 value; it is then formed in Python integers and saturated to the
    int64 range, which keeps the bucket: every threshold tau_k lies in [2, 2^63), so a saturated
    difference has the same count of thresholds <= max(dt, 1) as the exact one.
    """
    a = np.asarray(ts_q, np.int64).reshape(-1)
    b = np.asarray(ts_k, np.int64).reshape(-1)
    if a.size == 0 or b.size == 0:
        return np.zeros((a.size, b.size), np.int64)
    hi = int(a.max()) - int(b.min())
    lo = int(a.min()) - int(b.max())
    if -(2 ** 63) <= lo and hi < 2 ** 63:
        return a[:, None] - b[None, :]
    d = a.astype(object)[:, None] - b.astype(object)[None, :]
    d = np.minimum(np.maximum(d, -(2 ** 63)), 2 ** 63 - 1)
    return d.astype(np.int64)


def rel_pos_index(i, j, pos_max_len: int) -> np.ndarray:
    """Index into rab_pos for the pair (i, j): clip(i - j, -(L-1), L-1) + L - 1 (reading R6)."""
    L = int(pos_max_len)
    r = np.asarray(i, dtype=np.int64) - np.asarray(j, dtype=np.int64)
    return np.clip(r, -(L - 1), L - 1) + (L - 1)


# ----------------------------------------------------------------------------------------------
# Jagged metadata (the variable-length layout the efficiency paragraph's kernels work on)
# ----------------------------------------------------------------------------------------------

def seq_lengths(offsets: np.ndarray) -> np.ndarray:
    return np.diff(np.asarray(offsets, dtype=np.int64))


def tile_work_list(offsets: np.ndarray, block: int = 128) -> np.ndarray:
    """All (sequence b, query tile t) pairs, tile t covering local rows [t*block, (t+1)*block).

    Ordered by decreasing cost (a causal tile t visits t+1 key tiles), ties by increasing b.
    Returns int64 [n_items, 2] holding (b, t).
    """
    lens = seq_lengths(offsets)
    items = []
    for b, n in enumerate(lens):
        for t in range(-(-int(n) // block)):
            items.append((b, t))
    items.sort(key=lambda bt: (-bt[1], bt[0]))
    return np.array(items, dtype=np.int64).reshape(-1, 2)


# ----------------------------------------------------------------------------------------------
# Forward pieces of one HSTU layer
# ----------------------------------------------------------------------------------------------

def uvqk_fwd(x, W1, b1):
    """Z = X W1^T + b1 and S = SiLU(Z) (f1 then phi1; "Generative Recommenders and HSTU")."""
    x = np.asarray(x, np.float64)
    z = x @ np.asarray(W1, np.float64).T + np.asarray(b1, np.float64)
    return z, silu(z)


def split_uvqk(s, D: int):
    """Split S into the column blocks U | V | Q | K, in that order (the sketch's chunk order)."""
    return s[:, 0:D], s[:, D:2 * D], s[:, 2 * D:3 * D], s[:, 3 * D:4 * D]


def pair_bias(ts_q, ts_k, pos_q, pos_k, rab_pos, rab_time, pos_max_len, thresholds):
    """rab^{p,t}(i, j) = rab_pos[idx(p_i - p_j)] + rab_time[bucket(t_i - t_j)] for all pairs."""
    pi = np.asarray(pos_q, np.int64)[:, None]
    pj = np.asarray(pos_k, np.int64)[None, :]
    dt = time_diff(ts_q, ts_k)
    rp = np.asarray(rab_pos, np.float64)
    rt = np.asarray(rab_time, np.float64)
    return rp[rel_pos_index(pi, pj, pos_max_len)] + rt[time_bucket(dt, thresholds)]


def pointwise_attention_fwd(q, k, v, offsets, timestamps, rab_pos, rab_time, inv_N,
                            pos_max_len, thresholds, rows: Optional[Sequence[int]] = None):
    """O_i = sum_{j <= i, same sequence} SiLU(q_i . k_j + rab(i, j)) * inv_N * v_j, per head.

    q, k: [T, H, dqk]; v: [T, H, dv]; returns O [T, H, dv] (float64). When ``rows`` is given,
    only those global rows are evaluated and the others are NaN.

    "4.4 Scaling Recommendation Models", HSTU layer second equation and the pointwise-aggregation
    bullet; "HSTU: The First Exploration of the Scaling Law", 7.1.4 Innovation 1 (SiLU, no
    softmax, no 1/sqrt(d) scale); causal mask and division by a constant as in the sketch.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    T, H, _ = q.shape
    out = np.full((T, H, v.shape[2]), np.nan if rows is not None else 0.0)
    want = None if rows is None else np.zeros(T, bool)
    if want is not None:
        want[np.asarray(rows, np.int64)] = True
    for b in range(len(offsets) - 1):
        s, e = int(offsets[b]), int(offsets[b + 1])
        n = e - s
        if n == 0:
            continue
        local = np.arange(n) if want is None else np.nonzero(want[s:e])[0]
        if local.size == 0:
            continue
        # rows of this sequence are evaluated in groups only to bound memory
        for g0 in range(0, local.size, 512):
            li = local[g0:g0 + 512]
            nk = int(li.max()) + 1                     # keys j <= max(i) suffice (causal)
            lj = np.arange(nk)
            bias = pair_bias(timestamps[s + li], timestamps[s:s + nk], li, lj,
                             rab_pos, rab_time, pos_max_len, thresholds)
            causal = lj[None, :] <= li[:, None]
            for h in range(H):
                p = q[s + li, h, :] @ k[s:s + nk, h, :].T + bias
                a = np.where(causal, silu(p) * inv_N, 0.0)
                out[s + li, h, :] = a @ v[s:s + nk, h, :]
    return out


def pair_bias_ext(ts_q, ts_k, pos_q, pos_k, type_q, type_k, rab_pos_h, rab_time_h, rab_type_h, pos_max_len,
                  thresholds):
    """f(p_i - p_j, t_i - t_j, type_i, type_j) with one head's tables (reading R12):
    rab_pos_h[idx(p_i - p_j)] + rab_time_h[bucket(t_i - t_j)] + rab_type_h[type_i, type_j]; the type
    term is left out when rab_type_h is None."""
    b = pair_bias(ts_q, ts_k, pos_q, pos_k, rab_pos_h, rab_time_h, pos_max_len, thresholds)
    if rab_type_h is not None:
        tt = np.asarray(rab_type_h, np.float64)
        b = b + tt[np.asarray(type_q, np.int64)[:, None], np.asarray(type_k, np.int64)[None, :]]
    return b


def pointwise_attention_fwd_ext(q, k, v, offsets, timestamps, rab_pos, rab_time, inv_N, pos_max_len,
                                thresholds, token_type=None, rab_type=None, per_head=False):
    """The pointwise attention of ``pointwise_attention_fwd`` with the bias of reading R12: with
    per_head, rab_pos [H, 2L-1], rab_time [H, nb] and rab_type [H, nt, nt] give head h its own
    slices, else they are shared ([2L-1], [nb], [nt, nt]); token_type [T] holds each token's type
    (needed with rab_type)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    T, H, _ = q.shape
    out = np.zeros((T, H, v.shape[2]))
    ty = None if token_type is None else np.asarray(token_type, np.int64)
    for b in range(len(offsets) - 1):
        s, e = int(offsets[b]), int(offsets[b + 1])
        if e == s:
            continue
        li = np.arange(e - s)
        causal = li[None, :] <= li[:, None]
        for h in range(H):
            sl = (lambda t: None if t is None else np.asarray(t, np.float64)[h]) if per_head else \
                (lambda t: None if t is None else np.asarray(t, np.float64))
            bias = pair_bias_ext(timestamps[s:e], timestamps[s:e], li, li,
                                 None if ty is None else ty[s:e], None if ty is None else ty[s:e],
                                 sl(rab_pos), sl(rab_time), sl(rab_type), pos_max_len, thresholds)
            p = q[s:e, h] @ k[s:e, h].T + bias
            a = np.where(causal, silu(p) * inv_N, 0.0)
            out[s:e, h] = a @ v[s:e, h]
    return out


def pointwise_attention_bwd_ext(q, k, v, do, offsets, timestamps, rab_pos, rab_time, inv_N, pos_max_len,
                                thresholds, token_type=None, rab_type=None, per_head=False):
    """Gradients of ``pointwise_attention_fwd_ext``: dq, dk, dv and the gradients of rab_pos,
    rab_time and rab_type (same shapes as the tables; None for an absent rab_type). Each table
    entry receives dP of every pair (of every head sharing it) that reads it."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    do = np.asarray(do, np.float64)
    T, H, _ = q.shape
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    drp = np.zeros(np.asarray(rab_pos).shape)
    drt = np.zeros(np.asarray(rab_time).shape)
    dty = None if rab_type is None else np.zeros(np.asarray(rab_type).shape)
    ty = None if token_type is None else np.asarray(token_type, np.int64)
    for b in range(len(offsets) - 1):
        s, e = int(offsets[b]), int(offsets[b + 1])
        if e == s:
            continue
        li = np.arange(e - s)
        causal = li[None, :] <= li[:, None]
        pidx = rel_pos_index(li[:, None], li[None, :], pos_max_len)
        tidx = time_bucket(time_diff(timestamps[s:e], timestamps[s:e]), thresholds)
        for h in range(H):
            sl = (lambda t: None if t is None else np.asarray(t, np.float64)[h]) if per_head else \
                (lambda t: None if t is None else np.asarray(t, np.float64))
            bias = pair_bias_ext(timestamps[s:e], timestamps[s:e], li, li,
                                 None if ty is None else ty[s:e], None if ty is None else ty[s:e],
                                 sl(rab_pos), sl(rab_time), sl(rab_type), pos_max_len, thresholds)
            p = q[s:e, h] @ k[s:e, h].T + bias
            a = np.where(causal, silu(p) * inv_N, 0.0)
            dv[s:e, h] = a.T @ do[s:e, h]
            dp = np.where(causal, (do[s:e, h] @ v[s:e, h].T) * silu_grad(p) * inv_N, 0.0)
            dq[s:e, h] = dp @ k[s:e, h]
            dk[s:e, h] = dp.T @ q[s:e, h]
            tp = drp[h] if per_head else drp
            tt = drt[h] if per_head else drt
            np.add.at(tp, pidx[causal], dp[causal])
            np.add.at(tt, tidx[causal], dp[causal])
            if dty is not None:
                ti = np.broadcast_to(ty[s:e][:, None], (e - s, e - s))
                tj = np.broadcast_to(ty[s:e][None, :], (e - s, e - s))
                np.add.at(dty[h] if per_head else dty, (ti[causal], tj[causal]), dp[causal])
    return dq, dk, dv, drp, drt, dty


def norm_gate_fwd(o, u, gamma, beta, eps: float = LN_EPS):
    """G = (gamma * (O - mu) / sqrt(var + eps) + beta) (.) U over the full d_model of a token.

    "4.4 Scaling Recommendation Models", third equation Norm(AV) (.) U and the gating bullet;
    "HSTU: The First Exploration of the Scaling Law", 7.1.4 Innovation 3. Returns (G, mu, rstd).
    """
    o = np.asarray(o, np.float64)
    mu = o.mean(axis=1)
    var = ((o - mu[:, None]) ** 2).mean(axis=1)
    rstd = 1.0 / np.sqrt(var + eps)
    ln = (o - mu[:, None]) * rstd[:, None] * np.asarray(gamma, np.float64) \
        + np.asarray(beta, np.float64)
    return ln * np.asarray(u, np.float64), mu, rstd


def out_proj_fwd(g, W2, b2, x):
    """Y = G W2^T + b2 + X (f2 plus the residual, "Generative Recommenders and HSTU" / sketch)."""
    return (np.asarray(g, np.float64) @ np.asarray(W2, np.float64).T
            + np.asarray(b2, np.float64) + np.asarray(x, np.float64))


def layer_fwd(x, p, offsets, timestamps, H, inv_N, pos_max_len, thresholds, eps=LN_EPS,
              positions=None):
    """One HSTU layer: Y = f2(Norm(A V) (.) U) + X over jagged sequences.

    ``p`` has attributes W1, b1, W2, b2, gamma, beta, rab_pos, rab_time. Returns (Y, saved)
    where ``saved`` holds the intermediates the backward uses.
    """
    x = np.asarray(x, np.float64)
    T, D = x.shape
    d = D // H
    z, s = uvqk_fwd(x, p.W1, p.b1)
    u, v, q, k = split_uvqk(s, D)
    o = pointwise_attention_fwd(q.reshape(T, H, d), k.reshape(T, H, d), v.reshape(T, H, d),
                                offsets, timestamps, p.rab_pos, p.rab_time, inv_N, pos_max_len,
                                thresholds).reshape(T, D)
    g, mu, rstd = norm_gate_fwd(o, u, p.gamma, p.beta, eps)
    y = out_proj_fwd(g, p.W2, p.b2, x)
    return y, dict(x=x, z=z, s=s, o=o, g=g, mu=mu, rstd=rstd)


def layer_fwd_norm_in(x, p, gamma_in, beta_in, offsets, timestamps, H, inv_N, pos_max_len, thresholds,
                      eps=LN_EPS):
    """The variant of the first page's "Code" sketch that normalises the layer input first: f1 reads
    Xn = LayerNorm_in(X) (affine, over d_model, eps 1e-5), the residual adds X itself (the sketch
    returns x + f2(norm_av(av) * u) with u, v, q, k from f1(norm_in(x))). Returns (Y, saved) with
    saved["x"] = Xn, the LayerNorm_in statistics in saved["mu_in"], saved["rstd_in"] and the raw
    input in saved["x_raw"]."""
    x = np.asarray(x, np.float64)
    T, D = x.shape
    xn, mu_in, rstd_in = norm_gate_fwd(x, np.ones_like(x), gamma_in, beta_in, eps)
    d = D // H
    z, s = uvqk_fwd(xn, p.W1, p.b1)
    u, v, q, k = split_uvqk(s, D)
    o = pointwise_attention_fwd(q.reshape(T, H, d), k.reshape(T, H, d), v.reshape(T, H, d),
                                offsets, timestamps, p.rab_pos, p.rab_time, inv_N, pos_max_len,
                                thresholds).reshape(T, D)
    g, mu, rstd = norm_gate_fwd(o, u, p.gamma, p.beta, eps)
    y = out_proj_fwd(g, p.W2, p.b2, x)
    return y, dict(x=xn, z=z, s=s, o=o, g=g, mu=mu, rstd=rstd, x_raw=x, mu_in=mu_in, rstd_in=rstd_in)


# ----------------------------------------------------------------------------------------------
# Backward (closed form, derived from the forward equations; no autograd)
# ----------------------------------------------------------------------------------------------

def pointwise_attention_bwd(q, k, v, do, offsets, timestamps, rab_pos, rab_time, inv_N,
                            pos_max_len, thresholds):
    """Gradients of O = (SiLU(QK^T + rab) * inv_N, causal) V with respect to Q, K, V, rab_pos,
    rab_time. With A = SiLU(P) inv_N (masked): dV = A^T dO, dA = dO V^T,
    dP = dA * SiLU'(P) * inv_N (masked), dQ = dP K, dK = dP^T Q; the table gradients add dP of
    every head into the entry each pair reads.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    do = np.asarray(do, np.float64)
    T, H, _ = q.shape
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    drp = np.zeros(np.asarray(rab_pos).shape[0])
    drt = np.zeros(np.asarray(rab_time).shape[0])
    for b in range(len(offsets) - 1):
        s, e = int(offsets[b]), int(offsets[b + 1])
        n = e - s
        if n == 0:
            continue
        li = np.arange(n)
        bias = pair_bias(timestamps[s:e], timestamps[s:e], li, li, rab_pos, rab_time,
                         pos_max_len, thresholds)
        causal = li[None, :] <= li[:, None]
        pidx = rel_pos_index(li[:, None], li[None, :], pos_max_len)
        tidx = time_bucket(time_diff(timestamps[s:e], timestamps[s:e]), thresholds)
        dp_sum = np.zeros((n, n))
        for h in range(H):
            p = q[s:e, h] @ k[s:e, h].T + bias
            a = np.where(causal, silu(p) * inv_N, 0.0)
            dv[s:e, h] = a.T @ do[s:e, h]
            da = do[s:e, h] @ v[s:e, h].T
            dp = np.where(causal, da * silu_grad(p) * inv_N, 0.0)
            dq[s:e, h] = dp @ k[s:e, h]
            dk[s:e, h] = dp.T @ q[s:e, h]
            dp_sum += dp
        np.add.at(drp, pidx[causal], dp_sum[causal])
        np.add.at(drt, tidx[causal], dp_sum[causal])
    return dq, dk, dv, drp, drt


def norm_gate_bwd(dg, o, u, gamma, mu, rstd):
    """Backward of G = (gamma * xhat + beta) (.) U through the LayerNorm, xhat = (O - mu) rstd.

    Returns dO, dgamma, dbeta (dU = dG (.) (gamma * xhat + beta) is formed by the caller).
    """
    o = np.asarray(o, np.float64)
    xhat = (o - mu[:, None]) * rstd[:, None]
    dln = np.asarray(dg, np.float64) * np.asarray(u, np.float64)
    dgamma = (dln * xhat).sum(axis=0)
    dbeta = dln.sum(axis=0)
    dxhat = dln * np.asarray(gamma, np.float64)
    D = o.shape[1]
    do = rstd[:, None] * (dxhat - dxhat.sum(axis=1, keepdims=True) / D
                          - xhat * (dxhat * xhat).sum(axis=1, keepdims=True) / D)
    return do, dgamma, dbeta


def layer_bwd(dy, p, saved, offsets, timestamps, H, inv_N, pos_max_len, thresholds):
    """Closed-form backward of ``layer_fwd``. Returns dict of dX, dW1, db1, dW2, db2, dgamma,
    dbeta, drab_pos, drab_time (all float64)."""
    dy = np.asarray(dy, np.float64)
    x, z, s, o, g, mu, rstd = (saved[n] for n in ("x", "z", "s", "o", "g", "mu", "rstd"))
    T, D = x.shape
    d = D // H
    W1 = np.asarray(p.W1, np.float64)
    W2 = np.asarray(p.W2, np.float64)
    gamma = np.asarray(p.gamma, np.float64)
    beta = np.asarray(p.beta, np.float64)
    # f2 + residual
    dg = dy @ W2
    dW2 = dy.T @ g
    db2 = dy.sum(axis=0)
    # LN (.) U
    u, v, q, k = split_uvqk(s, D)
    xhat = (o - mu[:, None]) * rstd[:, None]
    ln = xhat * gamma + beta
    du = dg * ln
    do, dgamma, dbeta = norm_gate_bwd(dg, o, u, gamma, mu, rstd)
    # attention
    dq, dk, dv, drp, drt = pointwise_attention_bwd(
        q.reshape(T, H, d), k.reshape(T, H, d), v.reshape(T, H, d), do.reshape(T, H, d),
        offsets, timestamps, p.rab_pos, p.rab_time, inv_N, pos_max_len, thresholds)
    # f1 + SiLU
    ds = np.concatenate([du, dv.reshape(T, D), dq.reshape(T, D), dk.reshape(T, D)], axis=1)
    dz = ds * silu_grad(z)
    dW1 = dz.T @ x
    db1 = dz.sum(axis=0)
    dx = dy + dz @ W1
    return dict(dx=dx, dW1=dW1, db1=db1, dW2=dW2, db2=db2, dgamma=dgamma, dbeta=dbeta,
                drab_pos=drp, drab_time=drt, dz=dz, do=do)


def layer_bwd_norm_in(dy, p, gamma_in, saved, offsets, timestamps, H, inv_N, pos_max_len, thresholds):
    """Backward of ``layer_fwd_norm_in``: the layer's own gradients with Xn as f1's input (dW1 =
    dZ^T Xn), then d Xn = dZ W1 through LayerNorm_in back to X, dX = dY + LN_in^T(d Xn); also
    dgamma_in and dbeta_in."""
    r = layer_bwd(dy, p, saved, offsets, timestamps, H, inv_N, pos_max_len, thresholds)
    dxn = r["dz"] @ np.asarray(p.W1, np.float64)
    x = saved["x_raw"]
    dx_in, dgamma_in, dbeta_in = norm_gate_bwd(dxn, x, np.ones_like(x), gamma_in, saved["mu_in"],
                                               saved["rstd_in"])
    r = dict(r)
    r["dx"] = np.asarray(dy, np.float64) + dx_in
    r["dgamma_in"] = dgamma_in
    r["dbeta_in"] = dbeta_in
    return r


# ----------------------------------------------------------------------------------------------
# Stochastic Length ("HSTU: The First Exploration of the Scaling Law", 7.1.5)
# ----------------------------------------------------------------------------------------------

def stochastic_length_keep(n: int, alpha: float) -> int:
    """Number of tokens kept from a length-n history: min(n, floor(n**(alpha/2) + 1/2))."""
    return int(min(n, np.floor(float(n) ** (alpha / 2.0) + 0.5)))


def stochastic_length(offsets, keys, alpha: float):
    """Reading R10: keep, per sequence, the L tokens with the smallest keys (ties by position),
    in their original order. Returns (new_offsets int64 [B+1], kept global indices int64 [T'])."""
    offsets = np.asarray(offsets, np.int64)
    keys = np.asarray(keys, np.int64)
    new_off = [0]
    kept = []
    for b in range(len(offsets) - 1):
        s, e = int(offsets[b]), int(offsets[b + 1])
        n = e - s
        L = stochastic_length_keep(n, alpha)
        order = np.lexsort((np.arange(n), keys[s:e]))   # primary: key, secondary: position
        sel = np.sort(order[:L])
        kept.append(s + sel)
        new_off.append(new_off[-1] + L)
    kept_idx = np.concatenate(kept) if kept else np.zeros(0, np.int64)
    return np.array(new_off, np.int64), kept_idx.astype(np.int64)


# ----------------------------------------------------------------------------------------------
# M-FALCON ("HSTU: The First Exploration of the Scaling Law", 7.1.5 M-FALCON)
# ----------------------------------------------------------------------------------------------

def falcon_fwd(layers: List, prefix_offsets, prefix_ts, prefix_x, cand_x, request_ts, m: int,
               H: int, inv_N: float, pos_max_len: int, thresholds, eps=LN_EPS):
    """Score m candidates per user against the user's prefix, layer by layer (reading R11).

    Layer l: the prefix goes through the causal layer (its K, V are what a cache would hold);
    candidate c of user u uses keys = every prefix token j (relative position n - j, time
    difference request_ts[u] - t_j) plus itself (position difference 0, time difference 0).
    Candidates never see each other. Returns (candidate outputs [users*m, D], prefix outputs).
    """
    xp = np.asarray(prefix_x, np.float64)
    xc = np.asarray(cand_x, np.float64)
    D = xp.shape[1]
    d = D // H
    users = len(prefix_offsets) - 1
    for p in layers:
        yp, saved = layer_fwd(xp, p, prefix_offsets, prefix_ts, H, inv_N, pos_max_len,
                              thresholds, eps)
        sp = saved["s"]
        kp_all = sp[:, 3 * D:4 * D]
        vp_all = sp[:, D:2 * D]
        _, sc = uvqk_fwd(xc, p.W1, p.b1)
        uc, vc, qc, kc = split_uvqk(sc, D)
        oc = np.zeros((xc.shape[0], D))
        rp = np.asarray(p.rab_pos, np.float64)
        rt = np.asarray(p.rab_time, np.float64)
        for u_ in range(users):
            s, e = int(prefix_offsets[u_]), int(prefix_offsets[u_ + 1])
            n = e - s
            j = np.arange(n)
            bias_prefix = (rp[rel_pos_index(n, j, pos_max_len)]
                           + rt[time_bucket(time_diff([int(request_ts[u_])], prefix_ts[s:e])[0],
                                            thresholds)])
            bias_self = rp[rel_pos_index(0, 0, pos_max_len)] + rt[time_bucket(0, thresholds)]
            rows = slice(u_ * m, (u_ + 1) * m)
            for h in range(H):
                cs = slice(h * d, (h + 1) * d)
                sc_pre = qc[rows, cs] @ kp_all[s:e, cs].T + bias_prefix[None, :]
                sc_self = (qc[rows, cs] * kc[rows, cs]).sum(axis=1) + bias_self
                oc[rows, cs] = (silu(sc_pre) * inv_N) @ vp_all[s:e, cs] \
                    + (silu(sc_self) * inv_N)[:, None] * vc[rows, cs]
        gc, _, _ = norm_gate_fwd(oc, uc, p.gamma, p.beta, eps)
        yc = out_proj_fwd(gc, p.W2, p.b2, xc)
        xp, xc = yp, yc
    return xc, xp
