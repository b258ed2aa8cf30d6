"""Scalar brute-force evaluator of one HSTU layer: TEST INFRASTRUCTURE only.

Pure Python loops over (token, feature), (sequence, head, i, j) with ``math.exp`` and exact
``decimal`` logarithms for the time buckets, written independently of ``hstu_oracle`` (no shared
helper) so that it can pin that module on tiny inputs. Same readings R1-R9 as ``hstu_oracle`` (listed
in its header):
no input LayerNorm, constant 1/N, causal j <= i, tables shared by heads,
bucket = min(nb-1, floor(ln(max(dt,1))/0.301)), rab_pos index clip(i-j) + L - 1, U|V|Q|K split,
affine LayerNorm over d_model with eps 1e-5, residual after f2.
"""
from __future__ import annotations

import decimal
import math


def _silu(z: float) -> float:
    if z < -700.0:
        return 0.0
    return z / (1.0 + math.exp(-z))


def _bucket(dt: int, n_buckets: int) -> int:
    v = max(int(dt), 1)
    ctx = decimal.Context(prec=60)
    lnv = ctx.ln(decimal.Decimal(v))
    b = int((lnv / decimal.Decimal("0.301")).to_integral_value(rounding=decimal.ROUND_FLOOR))
    return min(n_buckets - 1, b)


def _pos(i: int, j: int, L: int) -> int:
    r = i - j
    if r > L - 1:
        r = L - 1
    if r < -(L - 1):
        r = -(L - 1)
    return r + L - 1


def layer_fwd_scalar(x, W1, b1, W2, b2, gamma, beta, rab_pos, rab_time, offsets, ts, H,
                     inv_N, L, eps=1e-5):
    """x: list of T rows of D floats; weights as nested lists. Returns Y as a list of rows."""
    T = len(x)
    D = len(x[0]) if T else 0
    d = D // H
    nb = len(rab_time)
    # f1 and SiLU, column blocks U | V | Q | K
    S = [[0.0] * (4 * D) for _ in range(T)]
    for t in range(T):
        for c in range(4 * D):
            acc = b1[c]
            for kk in range(D):
                acc += x[t][kk] * W1[c][kk]
            S[t][c] = _silu(acc)
    O = [[0.0] * D for _ in range(T)]
    for b in range(len(offsets) - 1):
        s0, s1 = offsets[b], offsets[b + 1]
        for i in range(s0, s1):
            for j in range(s0, i + 1):
                bias = rab_pos[_pos(i - s0, j - s0, L)] + rab_time[_bucket(ts[i] - ts[j], nb)]
                for h in range(H):
                    dot = 0.0
                    for c in range(d):
                        dot += S[i][2 * D + h * d + c] * S[j][3 * D + h * d + c]
                    a = _silu(dot + bias) * inv_N
                    for c in range(d):
                        O[i][h * d + c] += a * S[j][D + h * d + c]
    Y = []
    for t in range(T):
        mu = sum(O[t]) / D
        var = sum((o - mu) ** 2 for o in O[t]) / D
        rs = 1.0 / math.sqrt(var + eps)
        G = [((O[t][c] - mu) * rs * gamma[c] + beta[c]) * S[t][c] for c in range(D)]
        row = []
        for n in range(D):
            acc = b2[n] + x[t][n]
            for c in range(D):
                acc += G[c] * W2[n][c]
            row.append(acc)
        Y.append(row)
    return Y


def attention_scalar_ext(q, k, v, offsets, ts, types, rab_pos, rab_time, rab_type, per_head, inv_N, L):
    """Pointwise attention with the bias rab_pos[idx(i - j)] + rab_time[bucket(t_i - t_j)] +
    rab_type[type_i][type_j] (reading R12 of hstu_oracle), tables per head (per_head: nested lists
    indexed by head first) or shared; q, k, v: nested lists [T][H][d]; types: list of ints or None
    (no type term). Returns out [T][H][d]."""
    T = len(q)
    H = len(q[0]) if T else 0
    d = len(v[0][0]) if T else 0
    out = [[[0.0] * d for _ in range(H)] for _ in range(T)]
    for b in range(len(offsets) - 1):
        s0, s1 = offsets[b], offsets[b + 1]
        for i in range(s0, s1):
            for j in range(s0, i + 1):
                for h in range(H):
                    rp = rab_pos[h] if per_head else rab_pos
                    rt = rab_time[h] if per_head else rab_time
                    bias = rp[_pos(i - s0, j - s0, L)] + rt[_bucket(ts[i] - ts[j], len(rt))]
                    if types is not None:
                        ty = rab_type[h] if per_head else rab_type
                        bias += ty[types[i]][types[j]]
                    dot = 0.0
                    for c in range(len(q[i][h])):
                        dot += q[i][h][c] * k[j][h][c]
                    a = _silu(dot + bias) * inv_N
                    for c in range(d):
                        out[i][h][c] += a * v[j][h][c]
    return out
