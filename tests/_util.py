"""Shared helpers of the parity tests: tolerances and oracle calls on workloads."""
import numpy as np

from oracle import hstu_oracle as O

THR = O.time_bucket_thresholds(128)

# Tolerances. bf16 compute: |d| <= 1e-2 + 1e-2 |ref| on layer outputs. fp32 compute ("1e-4
# relative"): |d| <= 1e-4 + 1e-4 |ref|.
BF16_TOL = (1e-2, 1e-2)
F32_TOL = (1e-4, 1e-4)


def assert_close(actual, expected, atol, rtol, what=""):
    a = np.asarray(actual, np.float64)
    e = np.asarray(expected, np.float64)
    assert a.shape == e.shape, (what, a.shape, e.shape)
    assert np.all(np.isfinite(a)), f"{what}: non-finite values"
    err = np.abs(a - e)
    lim = atol + rtol * np.abs(e)
    bad = err > lim
    if bad.any():
        i = np.unravel_index(np.argmax(err - lim), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())}/{err.size} outside |d|<={atol}+{rtol}|ref|; "
                             f"worst at {i}: got {a[i]!r} expected {e[i]!r}")
    return float(err.max()) if err.size else 0.0


def layer_oracle(wl, layer_idx=0, x=None, rows=None):
    """Oracle layer forward of a workload (fp64), optionally only for selected output rows.

    With ``rows``, U|V|Q|K is computed for every token (keys of earlier positions are needed), the
    attention, norm-gate and f2 only for the selected rows. Returns (Y rows, dict of intermediates
    for those rows)."""
    p = wl.layers[layer_idx]
    x = wl.x if x is None else x
    T, D = x.shape
    d = D // wl.H
    z, s = O.uvqk_fwd(x, p.W1, p.b1)
    u, v, q, k = O.split_uvqk(s, D)
    o = O.pointwise_attention_fwd(q.reshape(T, wl.H, d), k.reshape(T, wl.H, d), v.reshape(T, wl.H, d),
                                  wl.offsets, wl.timestamps, p.rab_pos, p.rab_time, 1.0 / wl.N,
                                  wl.pos_max_len, THR, rows=rows).reshape(T, D)
    sel = np.arange(T) if rows is None else np.asarray(rows)
    g, mu, rstd = O.norm_gate_fwd(o[sel], u[sel], p.gamma, p.beta)
    y = O.out_proj_fwd(g, p.W2, p.b2, x[sel])
    return y, dict(z=z[sel], s=s[sel], o=o[sel], g=g, mu=mu, rstd=rstd)


def sample_rows(offsets, per_seq=6, seed=0):
    """A few rows of every sequence: first, last, tile edges and random ones."""
    rng = np.random.default_rng(seed)
    rows = []
    for b in range(len(offsets) - 1):
        s, e = int(offsets[b]), int(offsets[b + 1])
        n = e - s
        if n == 0:
            continue
        cand = {0, n - 1, min(n - 1, 127), min(n - 1, 128)}
        cand.update(int(r) for r in rng.integers(0, n, size=per_seq))
        rows.extend(s + r for r in sorted(cand))
    return np.array(sorted(set(rows)), np.int64)


# Canary guard words (a stand-in for an out-of-bounds checker, which this pool does not offer): the
# output tensor sits inside a larger allocation whose leading and trailing bytes hold a fixed pattern
# that no kernel may change.
CANARY = 0xA5


def guarded(shape, dtype, fill=float("nan"), guard_bytes=4096, device="cuda"):
    """(tensor, check): a device tensor of `shape` (filled with `fill`) between two guard regions of
    `guard_bytes` holding CANARY; check(what) asserts both regions are intact."""
    import torch
    elt = torch.empty((), dtype=dtype).element_size()
    n = int(np.prod(shape))
    g = guard_bytes // elt
    raw = torch.empty(n + 2 * g, dtype=dtype, device=device)
    raw.view(torch.uint8).fill_(CANARY)
    t = raw[g:g + n].view(*shape)
    if fill is not None:
        t.fill_(fill)

    def check(what=""):
        b = raw.view(torch.uint8)
        head, tail = b[:g * elt], b[(g + n) * elt:]
        assert bool((head == CANARY).all()), f"{what}: bytes before the output changed"
        assert bool((tail == CANARY).all()), f"{what}: bytes after the output changed"
    return t, check
