"""A rounding model of the CUDA path's 16-bit storage points: test infrastructure for the parity tests.

The tensor-core path keeps several intermediates in fp16 because the MMAs read 16-bit operands:
U|V|Q|K = SiLU(Z) and Z itself, the score s = q.k and the half bias 0.5 (rab_pos + rab_time) that
form the attention weight P in the forward, P itself, G = LN(O) (.) U, the upstream gradient dO of
the attention, the attention's P^T and dX (= dP) in the backward, and dZ before the dW1 / dX GEMMs;
a layer with an fp32 residual stream reads fp16 copies of X (f1, dW1) and of dY (dG, dW2). Every
accumulation is fp32 or wider.

This module evaluates a layer with the oracle's own steps (``oracle.hstu_oracle``) in float64 and
rounds the same values to fp16 at the same points. It is not an oracle: the oracle is exact. It
says how far from the oracle a correct implementation with those 16-bit operands lands, so that
the tests can (1) show on the CPU that the stated bf16 bound |d| <= 1e-2 + 1e-2 |ref| cannot hold
for every weight-gradient element when the attention's operands are 16-bit, and (2) hold the GPU's
count of elements outside that bound to a multiple of this model's count. The hardware's
approximate tanh (the SiLU of the f1 epilogue and of the attention weights) is not modelled; its
error is of the same order as one fp16 rounding.
"""
from __future__ import annotations

import numpy as np

from oracle import hstu_oracle as O

THR = O.time_bucket_thresholds(128)


def f16(a):
    return np.asarray(a, np.float64).astype(np.float16).astype(np.float64)


def _same(a):
    return np.asarray(a, np.float64)


# The storage points of the CUDA path, by name: "x" (fp16 copy of X for f1 and dW1), "uvqk", "z",
# "score" (q.k before the bias is added, forward), "bias" (the half bias), "p" (attention weights,
# both directions), "g", "dy" (fp16 copy of dY for dG and dW2), "do", "dx_attn" (dP), "dz".
ALL_POINTS = frozenset({"x", "uvqk", "z", "score", "bias", "p", "g", "dy", "do", "dx_attn", "dz"})


def rounder(points=ALL_POINTS):
    """r(name, a): a rounded to fp16 when `name` is one of `points`, else unchanged."""
    pts = frozenset(points)
    return lambda name, a: f16(a) if name in pts else _same(a)


def attention_fwd(q, k, v, off, ts, rab_pos, rab_time, inv_N, L, r=rounder()):
    """O = inv_N * sum_j P_ij v_j with P = r(SiLU(r(q.k) + bias)), bias = 2 r(0.5 rab)."""
    T, Hh, d = q.shape
    out = np.zeros((T, Hh, v.shape[2]))
    for b in range(len(off) - 1):
        s, e = int(off[b]), int(off[b + 1])
        if e == s:
            continue
        li = np.arange(e - s)
        bias = 2.0 * r("bias", 0.5 * O.pair_bias(ts[s:e], ts[s:e], li, li, rab_pos, rab_time, L, THR))
        causal = li[None, :] <= li[:, None]
        for h in range(Hh):
            p = np.where(causal, r("p", O.silu(r("score", q[s:e, h] @ k[s:e, h].T) + bias)), 0.0)
            out[s:e, h] = (p @ v[s:e, h]) * inv_N
    return out


def attention_bwd(q, k, v, do, off, ts, rab_pos, rab_time, inv_N, L, r=rounder()):
    """The backward with x = q.k + 2 r(0.5 rab) (fp32 score), P^T and dX rounded before the
    contractions that read them and before the head sum of the table gradients."""
    T, Hh, d = q.shape
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    drp, drt = np.zeros(len(rab_pos)), np.zeros(len(rab_time))
    for b in range(len(off) - 1):
        s, e = int(off[b]), int(off[b + 1])
        if e == s:
            continue
        li = np.arange(e - s)
        bias = 2.0 * r("bias", 0.5 * O.pair_bias(ts[s:e], ts[s:e], li, li, rab_pos, rab_time, L, THR))
        causal = li[None, :] <= li[:, None]
        pidx = O.rel_pos_index(li[:, None], li[None, :], L)
        tidx = O.time_bucket(O.time_diff(ts[s:e], ts[s:e]), THR)
        dsum = np.zeros((e - s, e - s))
        for h in range(Hh):
            x = q[s:e, h] @ k[s:e, h].T + bias
            p = np.where(causal, r("p", O.silu(x)), 0.0)
            dv[s:e, h] = (p.T @ do[s:e, h]) * inv_N
            dp = r("dx_attn", np.where(causal, (do[s:e, h] @ v[s:e, h].T) * O.silu_grad(x) * inv_N, 0.0))
            dq[s:e, h] = dp @ k[s:e, h]
            dk[s:e, h] = dp.T @ q[s:e, h]
            dsum += dp
        np.add.at(drp, pidx[causal], dsum[causal])
        np.add.at(drt, tidx[causal], dsum[causal])
    return dq, dk, dv, drp, drt


def layer_fwd(x, p, off, ts, H, inv_N, L, r=rounder(), x_f1=None):
    """Y and the saved intermediates; f1 reads r(x) (or x_f1 when given), the residual adds x itself."""
    x = _same(x)
    T, D = x.shape
    d = D // H
    z, s = O.uvqk_fwd(r("x", x) if x_f1 is None else x_f1, p.W1, p.b1)
    z, s = r("z", z), r("uvqk", s)
    u, v, q, k = O.split_uvqk(s, D)
    o = attention_fwd(q.reshape(T, H, d), k.reshape(T, H, d), v.reshape(T, H, d), off, ts, p.rab_pos,
                      p.rab_time, inv_N, L, r).reshape(T, D)
    g, mu, rstd = O.norm_gate_fwd(o, u, p.gamma, p.beta)
    g = r("g", g)
    y = O.out_proj_fwd(g, p.W2, p.b2, x)
    return y, dict(x=x if x_f1 is None else x_f1, z=z, s=s, o=o, g=g, mu=mu, rstd=rstd)


def layer_bwd(dy, p, sv, off, ts, H, inv_N, L, r=rounder()):
    """Gradients of one layer; dG and dW2 read r(dy), dX = dy + dZ W1 keeps dy itself."""
    dy = _same(dy)
    x, z, s, o, g, mu, rstd = (sv[n] for n in ("x", "z", "s", "o", "g", "mu", "rstd"))
    T, D = x.shape
    d = D // H
    dy16 = r("dy", dy)
    W1, W2 = _same(p.W1), _same(p.W2)
    gamma, beta = _same(p.gamma), _same(p.beta)
    dg = dy16 @ W2
    dW2 = dy16.T @ g
    db2 = dy.sum(axis=0)
    u, v, q, k = O.split_uvqk(s, D)
    ln = (o - mu[:, None]) * rstd[:, None] * gamma + beta
    du = dg * ln
    do, dgamma, dbeta = O.norm_gate_bwd(dg, o, u, gamma, mu, rstd)
    dq, dk, dv, drp, drt = attention_bwd(q.reshape(T, H, d), k.reshape(T, H, d), v.reshape(T, H, d),
                                         r("do", do).reshape(T, H, d), off, ts, p.rab_pos, p.rab_time, inv_N, L, r)
    ds = np.concatenate([du, dv.reshape(T, D), dq.reshape(T, D), dk.reshape(T, D)], axis=1)
    dz = r("dz", ds * O.silu_grad(z))
    return dict(dx=dy + dz @ W1, dz=dz, dW1=dz.T @ r("x", x), db1=dz.sum(axis=0), dW2=dW2, db2=db2, dgamma=dgamma,
                dbeta=dbeta, drab_pos=drp, drab_time=drt)


def layer_fwd_norm_in(x, p, gamma_in, beta_in, off, ts, H, inv_N, L, r=rounder()):
    """The norm_in variant: f1 reads Xn = LayerNorm_in(x) stored in fp16, the residual adds x."""
    x = _same(x)
    xn, mu, rstd = O.norm_gate_fwd(x, np.ones_like(x), gamma_in, beta_in)
    y, sv = layer_fwd(x, p, off, ts, H, inv_N, L, r, x_f1=r("x", xn))
    sv.update(x_raw=x, mu_in=mu, rstd_in=rstd)
    return y, sv


def layer_bwd_norm_in(dy, p, gamma_in, sv, off, ts, H, inv_N, L, r=rounder()):
    """Its backward: dW1 = dZ^T Xn (fp16 Xn), dXn = dZ W1 in fp32, dX = dY + LN_in^T(dXn)."""
    g = layer_bwd(dy, p, sv, off, ts, H, inv_N, L, r)
    dxn = g["dz"] @ _same(p.W1)
    x = sv["x_raw"]
    dx_in, dgi, dbi = O.norm_gate_bwd(dxn, x, np.ones_like(x), gamma_in, sv["mu_in"], sv["rstd_in"])
    g = dict(g)
    g.update(dx=_same(dy) + dx_in, dgamma_in=dgi, dbeta_in=dbi)
    return g


def stack_fwd_bwd(x, layers, off, ts, H, inv_N, L, dy, r=rounder()):
    """A stack of layers (residual stream kept at full width): (y, dx, per-layer gradient dicts)."""
    saved = []
    for p in layers:
        x, sv = layer_fwd(x, p, off, ts, H, inv_N, L, r)
        saved.append(sv)
    grads = [None] * len(layers)
    g = dy
    for i in reversed(range(len(layers))):
        grads[i] = layer_bwd(g, layers[i], saved[i], off, ts, H, inv_N, L, r)
        g = grads[i]["dx"]
    return x, g, grads


def misses(got, ref):
    """Elements outside the stated bf16 bound |d| <= 1e-2 + 1e-2 |ref|."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return int((np.abs(got - ref) > 1e-2 + 1e-2 * np.abs(ref)).sum())


def miss_ceiling(model_misses: int, size: int) -> int:
    """What the GPU may miss: twice the model's count (the unmodelled hardware tanh adds errors of
    the same order), plus 8 elements and one in 2,000 for the noise of counts that are small."""
    return 2 * model_misses + 8 + size // 2000
