"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Every function of ``oracle.hstu_oracle`` is checked here by at least one of: hand-worked values
(``tests/golden``), exact arithmetic, a scalar brute-force evaluator written independently,
closed forms, invariants (causality, jagged independence), a library routine (torch's
LayerNorm and dense ops for the page's dense formulation) and central finite differences.
"""
import decimal
import math
import os

import numpy as np
import pytest
import torch
from hypothesis import given, settings, strategies as st

from oracle import hstu_oracle as O
from oracle.bruteforce import layer_fwd_scalar
from hstu_sequential_transduction_causal_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
THR = O.time_bucket_thresholds(128)


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        rows = [ln for ln in f if ln.strip() and not ln.startswith("#")]
    return [float(v) for v in rows[0].split()]


# ---------------------------------------------------------------------------------------------
# time buckets and position indices
# ---------------------------------------------------------------------------------------------

def test_threshold_head_matches_hand_values():
    assert list(THR[:12]) == [int(v) for v in _golden("time_bucket_thresholds_head.txt")]


def test_bucket_matches_decimal_logarithm():
    rng = np.random.default_rng(1)
    vals = np.concatenate([np.arange(-3, 5000), rng.integers(5000, 2 ** 62, 3000),
                           (2 ** rng.uniform(0, 62, 3000)).astype(np.int64)])
    got = O.time_bucket(vals, THR)
    ctx = decimal.Context(prec=60)
    for v, g in zip(vals[::7], got[::7]):
        ln = ctx.ln(decimal.Decimal(max(int(v), 1)))
        ref = int((ln / decimal.Decimal("0.301")).to_integral_value(decimal.ROUND_FLOOR))
        assert g == min(127, ref), (v, g, ref)
    # the bulk against float64 logs, where the float value is far from an integer
    f = np.log(np.maximum(vals, 1).astype(np.float64)) / 0.301
    safe = np.abs(f - np.round(f)) > 1e-9
    assert np.array_equal(got[safe], np.minimum(127, np.floor(f[safe])).astype(np.int64))


def test_bucket_threshold_edges():
    for k in range(1, 128):
        t = int(THR[k - 1])
        assert O.time_bucket(t, THR) >= k
        assert O.time_bucket(t - 1, THR) <= k - 1
    assert O.time_bucket(-10 ** 12, THR) == 0
    assert O.time_bucket(0, THR) == 0 and O.time_bucket(1, THR) == 0
    assert O.time_bucket(2 ** 63 - 1, THR) == 127
    # bucket 1 is empty: tau_1 == tau_2 == 2
    assert O.time_bucket(2, THR) == 2


def test_rel_pos_index():
    L = 8
    assert O.rel_pos_index(5, 5, L) == L - 1
    assert O.rel_pos_index(7, 0, L) == 2 * L - 2
    assert O.rel_pos_index(100, 0, L) == 2 * L - 2      # clamped
    assert O.rel_pos_index(0, 3, L) == L - 1 - 3
    assert O.rel_pos_index(0, 100, L) == 0


# ---------------------------------------------------------------------------------------------
# activation
# ---------------------------------------------------------------------------------------------

def test_silu_values_and_gradient():
    assert O.silu(0.0) == 0.0
    assert abs(O.silu(1.0) - 0.7310585786300049) < 1e-15          # sigma(1)
    assert abs(O.silu(50.0) - 50.0) < 1e-12 and abs(O.silu(-50.0)) < 1e-18
    z = np.linspace(-8, 8, 101)
    h = 1e-6
    fd = (O.silu(z + h) - O.silu(z - h)) / (2 * h)
    assert np.allclose(O.silu_grad(z), fd, atol=1e-8)


# ---------------------------------------------------------------------------------------------
# layer forward: brute force, closed forms, invariants, page's dense formulation
# ---------------------------------------------------------------------------------------------

def _tiny(lengths, D=8, H=2, seed=3, L=16, spread=False):
    rng = np.random.default_rng(seed)
    wl = W.make_workload("c1", seed=seed, lengths=lengths, D=D, H=H, pos_max_len=L, N=L)
    p = wl.layers[0]
    # non-zero biases / affine so that every term is exercised
    p.b1 = rng.standard_normal(4 * D).astype(np.float32) * 0.3
    p.b2 = rng.standard_normal(D).astype(np.float32) * 0.3
    p.gamma = (1 + 0.3 * rng.standard_normal(D)).astype(np.float32)
    p.beta = (0.3 * rng.standard_normal(D)).astype(np.float32)
    p.rab_pos = rng.standard_normal(2 * L - 1).astype(np.float32)
    p.rab_time = rng.standard_normal(128).astype(np.float32)
    if spread:   # time gaps spanning many buckets, some equal and some out of order
        wl.timestamps = (wl.timestamps + rng.integers(-5, 10 ** 9, wl.T)).astype(np.int64)
    return wl, p


@pytest.mark.parametrize("spread", [False, True])
def test_layer_matches_scalar_bruteforce(spread):
    wl, p = _tiny([1, 3, 0, 5, 2], spread=spread)
    inv_N = 1.0 / 7.0
    y, _ = O.layer_fwd(wl.x, p, wl.offsets, wl.timestamps, wl.H, inv_N, wl.pos_max_len, THR)
    yb = layer_fwd_scalar(wl.x.astype(float).tolist(), p.W1.astype(float).tolist(),
                          p.b1.tolist(), p.W2.astype(float).tolist(), p.b2.tolist(),
                          p.gamma.tolist(), p.beta.tolist(), p.rab_pos.tolist(),
                          p.rab_time.tolist(), wl.offsets.tolist(), wl.timestamps.tolist(),
                          wl.H, inv_N, wl.pos_max_len)
    assert np.allclose(y, np.array(yb), rtol=1e-10, atol=1e-10)


def test_layer_matches_scalar_bruteforce_extreme_timestamps():
    """Timestamps near both ends of the int64 range: differences of up to 2^64 - 1, which have no
    int64 value, must still give the bucket of the true difference (the scalar loops subtract
    Python integers exactly)."""
    wl, p = _tiny([4, 3, 2])
    big = 2 ** 63 - 1
    wl.timestamps = np.array([-(2 ** 63), -5, 2 ** 62, big,       # spans of 2^63 + 2^62 and 2^64 - 1
                              big, -(2 ** 63), 0,                  # out of order, negative differences
                              big - 40, big], np.int64)
    inv_N = 0.5
    y, _ = O.layer_fwd(wl.x, p, wl.offsets, wl.timestamps, wl.H, inv_N, wl.pos_max_len, THR)
    yb = layer_fwd_scalar(wl.x.astype(float).tolist(), p.W1.astype(float).tolist(),
                          p.b1.tolist(), p.W2.astype(float).tolist(), p.b2.tolist(),
                          p.gamma.tolist(), p.beta.tolist(), p.rab_pos.tolist(),
                          p.rab_time.tolist(), wl.offsets.tolist(), [int(t) for t in wl.timestamps],
                          wl.H, inv_N, wl.pos_max_len)
    assert np.allclose(y, np.array(yb), rtol=1e-10, atol=1e-10)
    ts = [int(t) for t in wl.timestamps[:4]]
    exp = [[min(127, max(0, _decimal_bucket(a - b))) for b in ts] for a in ts]
    assert np.array_equal(O.time_bucket(O.time_diff(ts, ts), THR), np.array(exp))


def _decimal_bucket(dt):
    ctx = decimal.Context(prec=60)
    ln = ctx.ln(decimal.Decimal(max(int(dt), 1)))
    return int((ln / decimal.Decimal("0.301")).to_integral_value(decimal.ROUND_FLOOR))


@settings(max_examples=25, deadline=None, derandomize=True)
@given(lengths=st.lists(st.integers(0, 700), min_size=1, max_size=5), H=st.sampled_from([1, 3]),
       seed=st.integers(0, 2 ** 16), frac=st.sampled_from([0.02, 0.3, 1.0]))
def test_attention_row_subset_equals_full_evaluation(lengths, H, seed, frac):
    """``rows=`` groups the selected rows (by 512) and reads keys up to the group's last row; every
    selected row must equal the full evaluation's (up to the last bits of the matrix products,
    whose blocking depends on their shapes: a wrong key range or grouping moves rows by O(1)), and
    every other row must be NaN."""
    rng = np.random.default_rng(seed)
    off = W.offsets_from_lengths(lengths)
    T, d, L = int(off[-1]), 4, 300
    ts = W.draw_timestamps(rng, lengths)
    q, k, v = (rng.standard_normal((T, H, d)) for _ in range(3))
    rp, rt = rng.standard_normal(2 * L - 1), rng.standard_normal(128)
    full = O.pointwise_attention_fwd(q, k, v, off, ts, rp, rt, 1 / 64, L, THR)
    rows = np.nonzero(rng.random(T) < frac)[0]
    part = O.pointwise_attention_fwd(q, k, v, off, ts, rp, rt, 1 / 64, L, THR, rows=rows)
    assert np.allclose(part[rows], full[rows], rtol=1e-12, atol=1e-12)
    rest = np.setdiff1d(np.arange(T), rows)
    assert np.all(np.isnan(part[rest]))


@settings(max_examples=40, deadline=None, derandomize=True)
@given(lengths=st.lists(st.integers(0, 9), min_size=1, max_size=4), L=st.integers(2, 6),
       H=st.sampled_from([1, 2]), dh=st.sampled_from([2, 3]), seed=st.integers(0, 2 ** 16), spread=st.booleans(),
       inv_N=st.sampled_from([1.0, 0.25, 1.0 / 9.0]))
def test_layer_matches_scalar_bruteforce_random_shapes(lengths, L, H, dh, seed, spread, inv_N):
    """Seeded random shapes: empty and single-token sequences, one or two heads, odd head widths,
    and position tables shorter than the sequences, so that the relative-position clamp at +-(L-1)
    is taken in both the oracle and the scalar loops."""
    wl, p = _tiny(lengths, D=H * dh, H=H, seed=seed, L=L, spread=spread)
    y, _ = O.layer_fwd(wl.x, p, wl.offsets, wl.timestamps, wl.H, inv_N, wl.pos_max_len, THR)
    yb = layer_fwd_scalar(wl.x.astype(float).tolist(), p.W1.astype(float).tolist(),
                          p.b1.tolist(), p.W2.astype(float).tolist(), p.b2.tolist(),
                          p.gamma.tolist(), p.beta.tolist(), p.rab_pos.tolist(),
                          p.rab_time.tolist(), wl.offsets.tolist(), wl.timestamps.tolist(),
                          wl.H, inv_N, wl.pos_max_len)
    assert np.allclose(y, np.array(yb).reshape(y.shape), rtol=1e-10, atol=1e-10)


def test_causality_later_tokens_do_not_leak():
    wl, p = _tiny([9, 6])
    y0, _ = O.layer_fwd(wl.x, p, wl.offsets, wl.timestamps, wl.H, 0.1, wl.pos_max_len, THR)
    x2 = wl.x.copy()
    ts2 = wl.timestamps.copy()
    i = 4                                         # perturb tokens 5..8 of sequence 0
    x2[i + 1:9] += 3.0
    ts2[i + 1:9] += 123456
    y1, _ = O.layer_fwd(x2, p, wl.offsets, ts2, wl.H, 0.1, wl.pos_max_len, THR)
    assert np.array_equal(y0[:i + 1], y1[:i + 1])
    assert np.array_equal(y0[9:], y1[9:])
    assert not np.allclose(y0[i + 1:9], y1[i + 1:9])


def test_jagged_independence():
    wl, p = _tiny([5, 0, 7, 3])
    y, _ = O.layer_fwd(wl.x, p, wl.offsets, wl.timestamps, wl.H, 0.2, wl.pos_max_len, THR)
    for b in range(wl.B):
        s, e = wl.offsets[b], wl.offsets[b + 1]
        if e == s:
            continue
        yb, _ = O.layer_fwd(wl.x[s:e], p, np.array([0, e - s]), wl.timestamps[s:e], wl.H, 0.2,
                            wl.pos_max_len, THR)
        # identical up to the BLAS's rounding order of the row-block GEMMs
        assert np.allclose(y[s:e], yb, rtol=1e-13, atol=1e-13)


def test_closed_form_zero_query_key():
    """Q = K = 0 and zero tables: A = SiLU(0)/N = 0, O = 0, LN(O) = beta, so
    Y = (beta (.) U) W2^T + b2 + X; with beta = b2 = 0 it is X exactly."""
    wl, p = _tiny([4, 6])
    D = wl.D
    p.W1 = p.W1.copy()
    p.W1[2 * D:] = 0
    p.b1 = p.b1.copy()
    p.b1[2 * D:] = 0
    p.rab_pos = np.zeros_like(p.rab_pos)
    p.rab_time = np.zeros_like(p.rab_time)
    y, sv = O.layer_fwd(wl.x, p, wl.offsets, wl.timestamps, wl.H, 0.3, wl.pos_max_len, THR)
    u = sv["s"][:, :D]
    assert np.array_equal(sv["o"], np.zeros_like(sv["o"]))
    ref = (p.beta.astype(float) * u) @ p.W2.astype(float).T + p.b2 + wl.x
    assert np.allclose(y, ref, rtol=1e-14, atol=1e-14)
    p.beta = np.zeros_like(p.beta)
    p.b2 = np.zeros_like(p.b2)
    y, _ = O.layer_fwd(wl.x, p, wl.offsets, wl.timestamps, wl.H, 0.3, wl.pos_max_len, THR)
    assert np.array_equal(y, wl.x.astype(np.float64))


def test_closed_form_single_token():
    rng = np.random.default_rng(5)
    H, d, L = 2, 4, 8
    q, k, v = (rng.standard_normal((1, H, d)) for _ in range(3))
    rp = rng.standard_normal(2 * L - 1)
    rt = rng.standard_normal(128)
    o = O.pointwise_attention_fwd(q, k, v, [0, 1], np.array([77]), rp, rt, 0.25, L, THR)
    for h in range(H):
        p_ = float(q[0, h] @ k[0, h]) + rp[L - 1] + rt[0]
        assert np.allclose(o[0, h], p_ / (1 + math.exp(-p_)) * 0.25 * v[0, h], rtol=1e-14)


def test_constant_v_hand_values():
    L = 4
    rp = np.zeros(2 * L - 1)
    rp[L - 1 + 0], rp[L - 1 + 1], rp[L - 1 + 2] = 0.5, 1.0, -1.0
    q = np.zeros((3, 1, 2))
    v = np.ones((3, 1, 2))
    o = O.pointwise_attention_fwd(q, q, v, [0, 3], np.array([0, 0, 0]), rp, np.zeros(128), 1.0,
                                  L, THR)
    exp = _golden("constant_v_n3.txt")
    for i in range(3):
        assert np.allclose(o[i, 0], exp[i], rtol=0, atol=1e-15)


def test_dense_formulation_of_the_first_page():
    """The first page's sketch formulates one padded sequence densely: a per-head [n, n]
    position bias, causal lower triangle, division by n, LayerNorm over d_model, gate with U,
    f2 and the residual (its extra input LayerNorm left out, reading R1 of oracle/hstu_oracle.py;
    no time bias).
    Restated here with torch CPU ops and torch's LayerNorm; the oracle must agree."""
    n, D, H, L = 12, 16, 2, 16
    rng = np.random.default_rng(11)
    wl = W.make_workload("c1", seed=2, lengths=[n], D=D, H=H, pos_max_len=L, N=n)
    p = wl.layers[0]
    p.rab_time = np.zeros(128, np.float32)
    p.rab_pos = rng.standard_normal(2 * L - 1).astype(np.float32)
    y, _ = O.layer_fwd(wl.x, p, wl.offsets, wl.timestamps, H, 1.0 / n, L, THR)

    x = torch.tensor(wl.x, dtype=torch.float64)[None]              # [1, n, D]
    f1 = torch.nn.Linear(D, 4 * D).double()
    f2 = torch.nn.Linear(D, D).double()
    with torch.no_grad():
        f1.weight.copy_(torch.tensor(p.W1))
        f1.bias.copy_(torch.tensor(p.b1))
        f2.weight.copy_(torch.tensor(p.W2))
        f2.bias.copy_(torch.tensor(p.b2))
    ii = torch.arange(n)[:, None]
    jj = torch.arange(n)[None, :]
    dense = torch.tensor(p.rab_pos, dtype=torch.float64)[(ii - jj).clamp(-(L - 1), L - 1) + L - 1]
    dense = dense[None].expand(H, n, n)                             # same bias for every head
    u, v, q, k = torch.nn.functional.silu(f1(x)).chunk(4, dim=-1)
    heads = lambda t: t.view(1, n, H, D // H).transpose(1, 2)
    sc = heads(q) @ heads(k).transpose(-1, -2) + dense
    a = torch.nn.functional.silu(sc).masked_fill(~torch.ones(n, n, dtype=torch.bool).tril(), 0) / n
    av = (a @ heads(v)).transpose(1, 2).reshape(1, n, D)
    ln = torch.nn.functional.layer_norm(av, (D,), torch.tensor(p.gamma, dtype=torch.float64),
                                        torch.tensor(p.beta, dtype=torch.float64), eps=1e-5)
    yt = (x + f2(ln * u))[0].detach().numpy()
    assert np.allclose(y, yt, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# backward: central finite differences of the oracle's own forward
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("lengths,L", [([3, 5, 1], 8), ([9, 4, 1], 3)])
def test_backward_matches_finite_differences(lengths, L):
    """Central differences for every gradient. The second case has sequences longer than the
    position table (L = 3), so many pairs share the clamped entry rab_pos[2L-2]; there every entry
    of rab_pos is checked."""
    wl, p = _tiny(lengths, D=8, H=2, seed=7, L=L, spread=True)
    inv_N = 0.5
    rng = np.random.default_rng(8)
    dy = rng.standard_normal((wl.T, wl.D))
    for name in ("W1", "b1", "W2", "b2", "gamma", "beta", "rab_pos", "rab_time"):
        setattr(p, name, getattr(p, name).astype(np.float64))
    x = wl.x.astype(np.float64)

    def loss(xx, pp):
        yy, _ = O.layer_fwd(xx, pp, wl.offsets, wl.timestamps, wl.H, inv_N, wl.pos_max_len, THR)
        return float((yy * dy).sum())

    y, sv = O.layer_fwd(x, p, wl.offsets, wl.timestamps, wl.H, inv_N, wl.pos_max_len, THR)
    g = O.layer_bwd(dy, p, sv, wl.offsets, wl.timestamps, wl.H, inv_N, wl.pos_max_len, THR)
    h = 1e-6
    checks = [("dx", None, x)] + [("d" + n, n, getattr(p, n)) for n in
                                  ("W1", "b1", "W2", "b2", "gamma", "beta", "rab_pos",
                                   "rab_time")]
    for gname, pname, arr in checks:
        flat = arr.reshape(-1)
        idx = rng.choice(flat.size, size=min(flat.size, 25), replace=False)
        if pname == "rab_time":
            used = np.unique(O.time_bucket(
                wl.timestamps[:, None] - wl.timestamps[None, :], THR))
            idx = np.union1d(idx[:5], used)
        if pname == "rab_pos":
            idx = np.arange(flat.size)
        for t in idx:
            old = flat[t]
            flat[t] = old + h
            lp = loss(x, p)
            flat[t] = old - h
            lm = loss(x, p)
            flat[t] = old
            fd = (lp - lm) / (2 * h)
            an = g[gname].reshape(-1)[t]
            assert abs(fd - an) <= 1e-6 + 1e-5 * abs(fd), (gname, t, fd, an)


@settings(max_examples=25, deadline=None, derandomize=True)
@given(lengths=st.lists(st.integers(0, 7), min_size=1, max_size=3), L=st.integers(2, 5), H=st.sampled_from([1, 2]),
       d=st.sampled_from([2, 3]), seed=st.integers(0, 2 ** 16))
def test_attention_backward_finite_differences_random_shapes(lengths, L, H, d, seed):
    """The attention backward alone against central differences of the attention forward, over
    random jagged shapes whose sequences may outrun the position table (clamped entries), with
    unsorted and widely spread timestamps: dq, dk, dv on sampled entries, every rab_pos entry and
    every rab_time entry a pair reads."""
    rng = np.random.default_rng(seed)
    off = W.offsets_from_lengths(lengths)
    T = int(off[-1])
    ts = rng.integers(-5, 10 ** 7, T).astype(np.int64)
    q, k, v, do = (0.7 * rng.standard_normal((T, H, d)) for _ in range(4))
    rp, rt = rng.standard_normal(2 * L - 1), rng.standard_normal(128)
    inv_N = 0.4

    def loss():
        return float((O.pointwise_attention_fwd(q, k, v, off, ts, rp, rt, inv_N, L, THR) * do).sum())

    grads = O.pointwise_attention_bwd(q, k, v, do, off, ts, rp, rt, inv_N, L, THR)
    used_buckets = set()
    for b in range(len(lengths)):
        tb = ts[off[b]:off[b + 1]]
        used_buckets |= set(np.unique(O.time_bucket(tb[:, None] - tb[None, :], THR)).tolist())
    h = 1e-6
    for arr, g, idx in ((q, grads[0], None), (k, grads[1], None), (v, grads[2], None),
                        (rp, grads[3], np.arange(rp.size)), (rt, grads[4], np.array(sorted(used_buckets), int))):
        flat, gflat = arr.reshape(-1), g.reshape(-1)
        if idx is None:
            idx = rng.choice(flat.size, size=min(flat.size, 6), replace=False) if flat.size else np.array([], int)
        for t in idx:
            old = flat[t]
            flat[t] = old + h
            lp = loss()
            flat[t] = old - h
            lm = loss()
            flat[t] = old
            fd = (lp - lm) / (2 * h)
            assert abs(fd - gflat[t]) <= 1e-6 + 1e-5 * abs(fd), (t, fd, gflat[t])


@settings(max_examples=25, deadline=None, derandomize=True)
@given(T=st.integers(1, 9), D=st.sampled_from([1, 2, 5, 16]), eps=st.sampled_from([1e-5, 1e-3, 0.5]),
       scale=st.sampled_from([1e-3, 1.0, 1e3]), seed=st.integers(0, 2 ** 16))
def test_norm_gate_matches_torch_layer_norm_and_autograd(T, D, eps, scale, seed):
    """LayerNorm (.) U and its backward against torch's own layer_norm and autograd in float64 on
    the CPU: a library routine written independently of the oracle's closed forms. Rows of very
    small and very large spread exercise eps; D = 1 makes xhat zero."""
    rng = np.random.default_rng(seed)
    o = scale * rng.standard_normal((T, D)) + rng.standard_normal((T, 1))
    u, dg = rng.standard_normal((T, D)), rng.standard_normal((T, D))
    gamma, beta = 1 + 0.3 * rng.standard_normal(D), 0.3 * rng.standard_normal(D)
    g, mu, rstd = O.norm_gate_fwd(o, u, gamma, beta, eps)
    do, dgamma, dbeta = O.norm_gate_bwd(dg, o, u, gamma, mu, rstd)

    to = torch.tensor(o, dtype=torch.float64, requires_grad=True)
    tg = torch.tensor(gamma, dtype=torch.float64, requires_grad=True)
    tb = torch.tensor(beta, dtype=torch.float64, requires_grad=True)
    ln = torch.nn.functional.layer_norm(to, (D,), tg, tb, eps)
    ref = ln * torch.tensor(u, dtype=torch.float64)
    ref.backward(torch.tensor(dg, dtype=torch.float64))
    assert np.allclose(g, ref.detach().numpy(), rtol=1e-12, atol=1e-12)
    for got, want in ((do, to.grad), (dgamma, tg.grad), (dbeta, tb.grad)):
        w = want.numpy()
        assert np.allclose(got, w, rtol=1e-9, atol=1e-9 * max(1.0, float(np.abs(w).max()))), (got, w)


# ---------------------------------------------------------------------------------------------
# M-FALCON, Stochastic Length, work list
# ---------------------------------------------------------------------------------------------

def _check_falcon_against_naive(fw):
    """Candidate c of user u must equal the last row of a plain causal stack run on the user's
    prefix followed by that one candidate (timestamp = the request time), and the prefix outputs
    the other rows."""
    yc, yp = O.falcon_fwd(fw.layers, fw.prefix_offsets, fw.prefix_ts, fw.prefix_x, fw.cand_x,
                          fw.request_ts, fw.m, fw.H, 1 / fw.N, fw.pos_max_len, THR)
    for u in range(fw.users):
        s, e = fw.prefix_offsets[u], fw.prefix_offsets[u + 1]
        for c in range(fw.m):
            xs = np.concatenate([fw.prefix_x[s:e], fw.cand_x[u * fw.m + c][None]])
            ts = np.concatenate([fw.prefix_ts[s:e], [fw.request_ts[u]]])
            off = np.array([0, xs.shape[0]])
            for p in fw.layers:
                xs, _ = O.layer_fwd(xs, p, off, ts, fw.H, 1 / fw.N, fw.pos_max_len, THR)
            assert np.allclose(yc[u * fw.m + c], xs[-1], rtol=1e-12, atol=1e-12)
            assert np.allclose(yp[s:e], xs[:-1], rtol=1e-12, atol=1e-12)


def test_falcon_equals_naive_last_row():
    _check_falcon_against_naive(W.make_falcon_workload(seed=4, users=2, prefix=6, m=3, b_m=2, D=8, H=2,
                                                       layers=2, N=7, pos_max_len=8))


@settings(max_examples=20, deadline=None, derandomize=True)
@given(prefix_lengths=st.lists(st.integers(0, 7), min_size=1, max_size=3), m=st.integers(1, 3),
       L=st.integers(2, 9), layers=st.integers(1, 2), seed=st.integers(0, 2 ** 16))
def test_falcon_equals_naive_last_row_random_shapes(prefix_lengths, m, L, layers, seed):
    """Ragged prefixes (empty and single-token ones included) and position tables shorter than a
    prefix, so that a candidate's distance n - j to early prefix tokens is clamped as in a plain
    causal sequence."""
    _check_falcon_against_naive(W.make_falcon_workload(seed=seed, prefix_lengths=prefix_lengths, m=m, b_m=m,
                                                       D=8, H=2, layers=layers, N=7, pos_max_len=L))


def test_stochastic_length_counts_and_selection():
    assert O.stochastic_length_keep(512, 1.6) == 147       # 512**0.8 = 146.9
    assert O.stochastic_length_keep(4096, 1.6) == 776      # 2**9.6 = 776.05
    assert O.stochastic_length_keep(3, 1.6) == 2           # 3**0.8 = 2.41
    assert O.stochastic_length_keep(1, 1.6) == 1 and O.stochastic_length_keep(0, 1.6) == 0
    # n**0.8 is never within 1e-9 of a rounding boundary for the lengths the workloads draw
    n = np.arange(1, 10001, dtype=np.float64)
    f = n ** 0.8
    assert np.all(np.abs(f - np.floor(f) - 0.5) > 1e-9)
    rng = np.random.default_rng(0)
    lens = [0, 1, 5, 40, 17]
    off = W.offsets_from_lengths(lens)
    keys = rng.integers(0, 50, off[-1])                  # many ties on purpose
    new_off, kept = O.stochastic_length(off, keys, 1.6)
    for b, n_ in enumerate(lens):
        L = O.stochastic_length_keep(n_, 1.6)
        assert new_off[b + 1] - new_off[b] == L
        sel = kept[new_off[b]:new_off[b + 1]] - off[b]
        assert np.all(np.diff(sel) > 0)
        # brute force: a token is kept iff fewer than L tokens precede it in (key, position)
        for j in range(n_):
            rank = sum(1 for i in range(n_) if (keys[off[b] + i], i) < (keys[off[b] + j], j))
            assert (j in sel) == (rank < L)


@settings(max_examples=40, deadline=None, derandomize=True)
@given(lens=st.lists(st.integers(0, 60), min_size=0, max_size=6), alpha=st.sampled_from([1.2, 1.6, 2.0]),
       key_max=st.sampled_from([3, 1000, 2 ** 62]), seed=st.integers(0, 2 ** 16))
def test_stochastic_length_random_shapes(lens, alpha, key_max, seed):
    """Random jagged batches (empty ones included), few or many distinct keys: each sequence keeps
    exactly stochastic_length_keep(n) tokens, in order, and they are the lowest in (key, position)."""
    off = W.offsets_from_lengths(lens)
    keys = np.random.default_rng(seed).integers(0, key_max, off[-1], dtype=np.int64)
    new_off, kept = O.stochastic_length(off, keys, alpha)
    assert len(new_off) == len(lens) + 1 and new_off[0] == 0 and new_off[-1] == len(kept)
    for b, n_ in enumerate(lens):
        L = O.stochastic_length_keep(n_, alpha)
        sel = list(kept[new_off[b]:new_off[b + 1]] - off[b])
        order = sorted(range(n_), key=lambda i: (keys[off[b] + i], i))
        assert sel == sorted(order[:L])


@settings(max_examples=40, deadline=None, derandomize=True)
@given(lens=st.lists(st.integers(0, 700), min_size=0, max_size=8))
def test_work_list_random_shapes(lens):
    """Every (sequence, 128-row tile) once; longest remaining key range first, ties by sequence."""
    off = W.offsets_from_lengths(lens)
    wlst = O.tile_work_list(off, 128)
    expect = sorted(((b, t) for b, n in enumerate(lens) for t in range(-(-n // 128))), key=lambda r: (-r[1], r[0]))
    assert [tuple(int(v) for v in r) for r in wlst] == expect


def test_work_list_invariants():
    off = W.offsets_from_lengths([0, 1, 128, 129, 700, 256])
    wlst = O.tile_work_list(off, 128)
    expect = {(b, t) for b, n in enumerate(np.diff(off)) for t in range(-(-int(n) // 128))}
    assert {tuple(r) for r in wlst} == expect and len(wlst) == len(expect)
    for a, b in zip(wlst[:-1], wlst[1:]):
        assert a[1] > b[1] or (a[1] == b[1] and a[0] < b[0])


# ---------------------------------------------------------------------------------------------
# the richer bias: per-head tables and the token-type term (reading R12)
# ---------------------------------------------------------------------------------------------

def _ext_case(lengths, H=2, d=3, L=6, n_types=3, seed=0, spread=True):
    rng = np.random.default_rng(seed)
    off = W.offsets_from_lengths(lengths)
    T = int(off[-1])
    ts = W.draw_timestamps(rng, lengths)
    if spread:
        ts = (ts + rng.integers(-5, 10 ** 8, T)).astype(np.int64)
    q, k, v = (rng.standard_normal((T, H, d)) for _ in range(3))
    types = rng.integers(0, n_types, T)
    rp = rng.standard_normal((H, 2 * L - 1))
    rt = rng.standard_normal((H, 128))
    ty = rng.standard_normal((H, n_types, n_types))
    return off, ts, q, k, v, types, rp, rt, ty


@pytest.mark.parametrize("per_head,with_types", [(True, True), (True, False), (False, True)])
def test_attention_ext_matches_scalar_bruteforce(per_head, with_types):
    from oracle.bruteforce import attention_scalar_ext
    off, ts, q, k, v, types, rp, rt, ty = _ext_case([4, 0, 9, 1, 7], seed=5)
    if not per_head:
        rp, rt, ty = rp[0], rt[0], ty[0]
    inv_N = 0.2
    got = O.pointwise_attention_fwd_ext(q, k, v, off, ts, rp, rt, inv_N, 6, THR,
                                        token_type=types if with_types else None,
                                        rab_type=ty if with_types else None, per_head=per_head)
    exp = attention_scalar_ext(q.tolist(), k.tolist(), v.tolist(), off.tolist(), [int(t) for t in ts],
                               [int(t) for t in types] if with_types else None, rp.tolist(), rt.tolist(),
                               ty.tolist(), per_head, inv_N, 6)
    assert np.allclose(got, np.array(exp), rtol=1e-11, atol=1e-11)


def test_attention_ext_reduces_to_the_shared_tables():
    """Equal per-head slices and no type term give the shared-table attention; a type table holding
    one constant c everywhere gives the shared attention with c added to every rab_pos entry."""
    off, ts, q, k, v, types, rp, rt, ty = _ext_case([5, 11, 2], H=3, seed=7)
    base = O.pointwise_attention_fwd(q, k, v, off, ts, rp[0], rt[0], 0.3, 6, THR)
    same = O.pointwise_attention_fwd_ext(q, k, v, off, ts, np.repeat(rp[:1], 3, 0), np.repeat(rt[:1], 3, 0), 0.3, 6,
                                         THR, per_head=True)
    assert np.allclose(same, base, rtol=1e-13, atol=1e-13)
    c = 0.37
    shifted = O.pointwise_attention_fwd(q, k, v, off, ts, rp[0] + c, rt[0], 0.3, 6, THR)
    const = O.pointwise_attention_fwd_ext(q, k, v, off, ts, rp[0], rt[0], 0.3, 6, THR, token_type=types,
                                          rab_type=np.full((3, 3), c))
    assert np.allclose(const, shifted, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("per_head", [True, False])
def test_attention_ext_backward_finite_differences(per_head):
    off, ts, q, k, v, types, rp, rt, ty = _ext_case([3, 6, 1], H=2, d=2, L=4, seed=9)
    if not per_head:
        rp, rt, ty = rp[0], rt[0], ty[0]
    rng = np.random.default_rng(1)
    do = rng.standard_normal(q.shape)
    kw = dict(token_type=types, per_head=per_head)

    def loss(q_=q, k_=k, v_=v, rp_=rp, rt_=rt, ty_=ty):
        o = O.pointwise_attention_fwd_ext(q_, k_, v_, off, ts, rp_, rt_, 0.5, 4, THR, rab_type=ty_, **kw)
        return float(np.sum(o * do))

    dq, dk, dv, drp, drt, dty = O.pointwise_attention_bwd_ext(q, k, v, do, off, ts, rp, rt, 0.5, 4, THR,
                                                              rab_type=ty, **kw)
    eps = 1e-6
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv), ("rp", rp, drp), ("rt", rt, drt),
                            ("ty", ty, dty)):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            a1, a2 = arr.copy(), arr.copy()
            a1[idx] += eps
            a2[idx] -= eps
            fd[idx] = (loss(**{f"{name}_": a1}) - loss(**{f"{name}_": a2})) / (2 * eps)
        assert np.allclose(grad, fd, rtol=1e-5, atol=1e-7), name


# ---------------------------------------------------------------------------------------------
# the sketch's input LayerNorm (the norm_in variant of reading R1)
# ---------------------------------------------------------------------------------------------

def test_norm_in_variant_matches_the_first_page_sketch():
    """The first page's sketch with its input LayerNorm kept (f1 reads norm_in(x), the residual adds
    x), restated with torch ops and torch's LayerNorm, against layer_fwd_norm_in."""
    n, D, H, L = 10, 16, 2, 16
    rng = np.random.default_rng(12)
    wl = W.make_workload("c1", seed=4, lengths=[n], D=D, H=H, pos_max_len=L, N=n)
    p = wl.layers[0]
    p.rab_time = np.zeros(128, np.float32)
    p.rab_pos = rng.standard_normal(2 * L - 1).astype(np.float32)
    g_in, b_in = 1 + 0.3 * rng.standard_normal(D), 0.3 * rng.standard_normal(D)
    x_np = 3.0 + 2.0 * rng.standard_normal((n, D))          # far from normalised, so norm_in matters
    y, _ = O.layer_fwd_norm_in(x_np, p, g_in, b_in, wl.offsets, wl.timestamps, H, 1.0 / n, L, THR)
    x = torch.tensor(x_np, dtype=torch.float64)[None]
    f1 = torch.nn.Linear(D, 4 * D).double()
    f2 = torch.nn.Linear(D, D).double()
    with torch.no_grad():
        f1.weight.copy_(torch.tensor(p.W1))
        f1.bias.copy_(torch.tensor(p.b1))
        f2.weight.copy_(torch.tensor(p.W2))
        f2.bias.copy_(torch.tensor(p.b2))
    ii, jj = torch.arange(n)[:, None], torch.arange(n)[None, :]
    dense = torch.tensor(p.rab_pos, dtype=torch.float64)[(ii - jj).clamp(-(L - 1), L - 1) + L - 1][None].expand(H, n, n)
    xn = torch.nn.functional.layer_norm(x, (D,), torch.tensor(g_in), torch.tensor(b_in), eps=1e-5)
    u, v, q, k = torch.nn.functional.silu(f1(xn)).chunk(4, dim=-1)
    heads = lambda t: t.view(1, n, H, D // H).transpose(1, 2)
    sc = heads(q) @ heads(k).transpose(-1, -2) + dense
    a = torch.nn.functional.silu(sc).masked_fill(~torch.ones(n, n, dtype=torch.bool).tril(), 0) / n
    av = (a @ heads(v)).transpose(1, 2).reshape(1, n, D)
    ln = torch.nn.functional.layer_norm(av, (D,), torch.tensor(p.gamma, dtype=torch.float64),
                                        torch.tensor(p.beta, dtype=torch.float64), eps=1e-5)
    yt = (x + f2(ln * u))[0].detach().numpy()
    assert np.allclose(y, yt, rtol=1e-12, atol=1e-12)


def test_norm_in_backward_finite_differences():
    wl, p = _tiny([3, 4, 1], D=8, H=2, seed=6)
    rng = np.random.default_rng(3)
    x = 1.5 + rng.standard_normal((wl.T, wl.D))
    g_in, b_in = 1 + 0.3 * rng.standard_normal(wl.D), 0.3 * rng.standard_normal(wl.D)
    dy = rng.standard_normal((wl.T, wl.D))
    args = (wl.offsets, wl.timestamps, wl.H, 0.2, wl.pos_max_len, THR)

    def loss(x_=x, g_=g_in, b_=b_in, W1=None):
        pp = p if W1 is None else type(p)(**{**p.__dict__, "W1": W1})
        return float(np.sum(O.layer_fwd_norm_in(x_, pp, g_, b_, *args)[0] * dy))

    _, sv = O.layer_fwd_norm_in(x, p, g_in, b_in, *args)
    r = O.layer_bwd_norm_in(dy, p, g_in, sv, *args)
    eps = 1e-6
    for name, arr, grad, kw in (("dx", x, r["dx"], "x_"), ("dgamma_in", g_in, r["dgamma_in"], "g_"),
                                ("dbeta_in", b_in, r["dbeta_in"], "b_"), ("dW1", np.asarray(p.W1, np.float64),
                                                                          r["dW1"], "W1")):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            a1, a2 = arr.copy(), arr.copy()
            a1[idx] += eps
            a2[idx] -= eps
            fd[idx] = (loss(**{kw: a1}) - loss(**{kw: a2})) / (2 * eps)
        assert np.allclose(grad, fd, rtol=1e-5, atol=1e-7), name
