"""GPU parity of the forward path: each step and the whole layer, through the C ABI, against the
CPU oracle on the same seeded inputs. Integer work (work list, time buckets) is bit-exact;
floating outputs meet |d| <= 1e-2 + 1e-2|ref| (bf16) or 1e-4 + 1e-4|ref| (fp32)."""
import numpy as np
import pytest
import torch

from oracle import hstu_oracle as O
from hstu_sequential_transduction_causal_b200 import hstu as H
from hstu_sequential_transduction_causal_b200 import workloads as W
from hstu_sequential_transduction_causal_b200.runtime import (DeviceLayer, JaggedBatch, LayerRunner, to_dev,
                                                              workspace)
from tests._util import BF16_TOL, F32_TOL, THR, assert_close, layer_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from hstu_sequential_transduction_causal_b200 import build
    build.build()
    H.lib()
    torch.cuda.init()


def _bf16(a):
    return W.round_bf16(np.asarray(a, np.float64))


def _silu_like(rng, shape):
    z = rng.standard_normal(shape)
    return _bf16(z / (1 + np.exp(-z)))


# ---------------------------------------------------------------------------------------------
# integer steps: bit-exact
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("lengths", [
    [0, 1, 127, 128, 129, 300, 1024, 5, 0, 700, 256, 257],                     # one-warp path (B <= 32)
    [129 * (i % 7) + (i % 3) for i in range(32)],                              # one-warp path, B = 32
    [37 * i % 1025 for i in range(45)],                                        # block path (B > 32)
])
def test_worklist_bit_exact(lengths):
    off = W.offsets_from_lengths(lengths)
    jag = JaggedBatch(off, np.zeros(off[-1], np.int64), max_len=1024)
    cap = H.hstu_worklist_capacity(jag.struct)
    items = torch.full((cap, 2), -1, dtype=torch.int32, device="cuda")
    count = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    H.hstu_jagged_worklist(jag.struct, items, count)
    exp = O.tile_work_list(off, 128)
    n = int(count.item())
    assert n == len(exp)
    assert np.array_equal(items[:n].cpu().numpy().astype(np.int64), exp)


def _tile_paths(ts, off):
    """Which bucket arithmetic each 128 x 128 (query tile, key tile) of every sequence takes: the
    kernels use 32 bits when the tile's timestamps (query and key rows, rows past the end clamped
    to the last token) span less than 2^31 - 1, else the 64-bit path."""
    paths = set()
    for b in range(len(off) - 1):
        s, e = int(off[b]), int(off[b + 1])
        n = e - s
        nt = -(-n // 128)
        for qt in range(nt):
            for kt in range(nt):
                rows = [min(qt * 128 + r, n - 1) for r in range(128)] + [min(kt * 128 + c, n - 1) for c in range(128)]
                v = [int(ts[s + r]) for r in rows]
                paths.add("32" if max(v) - min(v) < 2 ** 31 - 1 else "64")
    return paths


def _bucket_surface(off, ts, max_len=None):
    jag = JaggedBatch(off, ts, max_len=max_len)
    lens = np.diff(off)
    sq = W.offsets_from_lengths(lens ** 2)
    out = torch.full((max(int(sq[-1]), 1),), 255, dtype=torch.uint8, device="cuda")
    H.hstu_time_buckets(jag.struct, 128, to_dev(sq, torch.int64), out)
    got = out.cpu().numpy()
    res = []
    for b in range(len(off) - 1):
        s, e = int(off[b]), int(off[b + 1])
        n = e - s
        res.append((got[sq[b]:sq[b + 1]].astype(np.int64).reshape(n, n),
                    O.time_bucket(O.time_diff(ts[s:e], ts[s:e]), THR)))
    return res


def test_time_buckets_bit_exact():
    rng = np.random.default_rng(3)
    lengths = [3, 70, 0, 200, 1, 300]
    off = W.offsets_from_lengths(lengths)
    ts = W.draw_timestamps(rng, lengths)
    # sequence 1: out of order, negative and threshold-adjacent differences, huge gaps
    s1 = slice(int(off[1]), int(off[2]))
    taus = THR[rng.integers(0, 127, size=70)]
    ts[s1] = 10 ** 15 + np.where(rng.random(70) < 0.5, taus, taus - 1) * rng.choice([-1, 1], 70)
    ts[int(off[3]):int(off[3]) + 5] = [0, 2 ** 62, -(2 ** 61), 7, 7]
    assert _tile_paths(ts, off) == {"32", "64"}
    for b, (got, exp) in enumerate(_bucket_surface(off, ts)):
        assert np.array_equal(got, exp), b


def test_time_buckets_every_threshold_edge_32_bit_path():
    """Differences tau_k - 1, tau_k, tau_k + 1 for every threshold below 2^31 (and 0, 1, 2), all in
    tiles whose timestamps span less than 2^31 - 1: the 32-bit path meets every bucket edge that an
    int32 difference can reach, from both sides, with positive and negative differences."""
    vals = [0, 1, 2]
    for t in THR:
        if int(t) + 1 < 2 ** 31 - 1:
            vals += [int(t) - 1, int(t), int(t) + 1]
    ts = np.array(vals, dtype=np.int64)
    off = np.array([0, len(ts)], np.int64)
    assert _tile_paths(ts, off) == {"32"}
    (got, exp), = _bucket_surface(off, ts)
    assert np.array_equal(got, exp)
    # every bucket an int32 difference can reach appears, and each edge is crossed
    assert set(np.unique(exp[:, 0])) >= set(range(2, 72)) - {1}
    assert np.array_equal(got[:, 0], O.time_bucket(ts, THR))


def test_time_buckets_every_threshold_edge_64_bit_path():
    """The same edges for every threshold, together with int64-sized gaps, so that the tiles holding
    the larger thresholds take the 64-bit path."""
    vals = [0, 1, 2]
    for t in THR:
        vals += [int(t) - 1, int(t), int(t) + 1]
    vals += [2 ** 40, 2 ** 55 + 3, 2 ** 62 - 1]
    ts = np.array(vals, dtype=np.int64)
    off = np.array([0, len(ts)], np.int64)
    assert _tile_paths(ts, off) == {"32", "64"}
    (got, exp), = _bucket_surface(off, ts)
    assert np.array_equal(got, exp)
    assert np.array_equal(got[:, 0], O.time_bucket(ts, THR))


def test_time_buckets_spans_around_2_31_and_int64_extremes():
    """Tile spans just under and at the 32-bit limit (2^31 - 2 takes 32 bits, 2^31 - 1 and 2^31 take
    64), and timestamps at both ends of the int64 range, whose differences (up to 2^64 - 1) have no
    int64 value: they must give the bucket of the true difference."""
    big = 2 ** 63 - 1
    seqs = [
        [0, 2 ** 31 - 2, 5, 2 ** 31 - 3],                 # span 2^31 - 2: 32-bit
        [0, 2 ** 31 - 1, 1, 2 ** 31 - 2],                 # span 2^31 - 1: 64-bit
        [2 ** 31, 0, 17, 2 ** 31 - 40],                   # span 2^31: 64-bit
        [-(2 ** 63), big, 0, -5, big - 1, -(2 ** 63) + 3, 2 ** 62],
        [big, big - 1, big - int(THR[126]), big - int(THR[126]) + 1, -(2 ** 63)],
    ]
    off = W.offsets_from_lengths([len(q) for q in seqs])
    ts = np.array([t for q in seqs for t in q], dtype=np.int64)
    paths = [_tile_paths(ts[int(off[b]):int(off[b + 1])], np.array([0, off[b + 1] - off[b]])) for b in range(5)]
    assert paths == [{"32"}, {"64"}, {"64"}, {"64"}, {"64"}]
    for b, (got, exp) in enumerate(_bucket_surface(off, ts)):
        assert np.array_equal(got, exp), b
    # the extreme pairs themselves: INT64_MAX - INT64_MIN lies above every threshold
    got3, _ = _bucket_surface(off, ts)[3]
    assert got3[1, 0] == 127 and got3[0, 1] == 0


# ---------------------------------------------------------------------------------------------
# single steps
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,act", [("bf16", "f16"), ("bf16", "bf16"), ("f32", "f32")])
def test_uvqk_fwd(dtype, act):
    rng = np.random.default_rng(1)
    T, D = (333, 256) if dtype == "bf16" else (437, 64)
    bf = dtype == "bf16"
    tdt = torch.bfloat16 if bf else torch.float32
    adt = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}[act]
    cast = _bf16 if bf else (lambda a: np.asarray(a, np.float32))
    x = cast(rng.standard_normal((T, D)))
    W1 = cast(rng.standard_normal((4 * D, D)) / np.sqrt(D))
    b1 = (0.1 * rng.standard_normal(4 * D)).astype(np.float32)
    uvqk = torch.empty(T, 4 * D, dtype=adt, device="cuda")
    z = torch.empty(T, 4 * D, dtype=adt, device="cuda")
    ws = workspace(256)
    H.hstu_uvqk_fwd(T, D, H.HSTU_BF16 if bf else H.HSTU_F32, H._dtype_code(uvqk), to_dev(x, tdt), D,
                    to_dev(W1, tdt), to_dev(b1, torch.float32), uvqk, z, ws)
    ze, se = O.uvqk_fwd(x, W1, b1)
    tol = BF16_TOL if bf else F32_TOL
    assert_close(z.float().cpu().numpy(), ze, *tol, what="Z")
    assert_close(uvqk.float().cpu().numpy(), se, *tol, what="SiLU(Z)")
    assert H.hstu_sync_status(ws) == 0


def _f16(a):
    return np.asarray(a, np.float64).astype(np.float16).astype(np.float32)


def _attn_case(lengths, Hh, d, L, inv_N, bf, seed=0, table_std=1.0, spread_ts=False, f16=False):
    rng = np.random.default_rng(seed)
    off = W.offsets_from_lengths(lengths)
    T = int(off[-1])
    ts = W.draw_timestamps(rng, lengths)
    if spread_ts:
        ts = ts + rng.integers(-10 ** 6, 10 ** 9, size=T)
    cast = (_f16 if f16 else _bf16) if bf else (lambda a: np.asarray(a, np.float32))
    q = _silu_like(rng, (T, Hh * d)) if bf else rng.standard_normal((T, Hh * d)).astype(np.float32)
    k = _silu_like(rng, (T, Hh * d)) if bf else rng.standard_normal((T, Hh * d)).astype(np.float32)
    v = _silu_like(rng, (T, Hh * d)) if bf else rng.standard_normal((T, Hh * d)).astype(np.float32)
    q, k, v = cast(q), cast(k), cast(v)
    rp = (table_std * rng.standard_normal(2 * L - 1)).astype(np.float32)
    rt = (table_std * rng.standard_normal(128)).astype(np.float32)
    return off, ts, q, k, v, rp, rt


def _run_attn(off, ts, q, k, v, rp, rt, Hh, d, L, inv_N, bf, max_len=None, out_bf16=False, f16=False):
    tdt = (torch.float16 if f16 else torch.bfloat16) if bf else torch.float32
    jag = JaggedBatch(off, ts, max_len=max_len)
    T = jag.T
    desc = H.make_attn_desc(Hh, d, d, inv_N, L, H._dtype_code(torch.empty(0, dtype=tdt)), Hh * d, Hh * d, Hh * d, Hh * d,
                            o_dtype_code=H.HSTU_BF16 if out_bf16 else H.HSTU_F32)
    ws = workspace(H.hstu_attn_workspace_size(desc, jag.struct))
    out = torch.full((T, Hh * d), float("nan"), dtype=torch.bfloat16 if out_bf16 else torch.float32,
                     device="cuda")
    H.hstu_attn_fwd(desc, jag.struct, to_dev(q, tdt), to_dev(k, tdt), to_dev(v, tdt), to_dev(rp, torch.float32),
                    to_dev(rt, torch.float32), out, ws)
    st = H.hstu_sync_status(ws)
    return out.float().cpu().numpy(), st


@pytest.mark.parametrize("spread,out_bf16,f16", [(False, False, True), (True, False, True), (False, True, False),
                                                  (True, False, False)])
def test_attn_fwd_tensor_core_ragged(spread, out_bf16, f16):
    lengths = [1, 127, 128, 129, 300, 0, 513, 64, 2]
    Hh, d, L = 2, 64, 600
    inv_N = 1.0 / 512
    off, ts, q, k, v, rp, rt = _attn_case(lengths, Hh, d, L, inv_N, True, seed=2, spread_ts=spread, f16=f16)
    got, st = _run_attn(off, ts, q, k, v, rp, rt, Hh, d, L, inv_N, True, out_bf16=out_bf16, f16=f16)
    assert st == 0
    T = int(off[-1])
    exp = O.pointwise_attention_fwd(q.reshape(T, Hh, d), k.reshape(T, Hh, d), v.reshape(T, Hh, d), off, ts, rp, rt,
                                    inv_N, L, THR).reshape(T, Hh * d)
    scale = float(np.sqrt(np.mean(exp ** 2)))
    # the attention output alone: |d| <= 1e-2 rms(ref) + 1e-2 |ref| (16-bit operands, fp32 accumulate)
    assert_close(got, exp, 1e-2 * scale, 1e-2, what="O")


def test_attn_fwd_tensor_core_odd_head_count():
    lengths = [130, 1, 385]
    Hh, d, L = 3, 64, 400
    inv_N = 1.0 / 300
    off, ts, q, k, v, rp, rt = _attn_case(lengths, Hh, d, L, inv_N, True, seed=7, f16=True)
    got, st = _run_attn(off, ts, q, k, v, rp, rt, Hh, d, L, inv_N, True, f16=True)
    assert st == 0
    T = int(off[-1])
    exp = O.pointwise_attention_fwd(q.reshape(T, Hh, d), k.reshape(T, Hh, d), v.reshape(T, Hh, d), off, ts, rp, rt,
                                    inv_N, L, THR).reshape(T, Hh * d)
    scale = float(np.sqrt(np.mean(exp ** 2)))
    assert_close(got, exp, 1e-2 * scale, 1e-2, what="O (3 heads)")


def test_attn_fwd_f32_single_layer_workload():
    wl = W.make_workload("c1", seed=0)
    Hh, d, L = wl.H, wl.D // wl.H, wl.pos_max_len
    off, ts, q, k, v, rp, rt = _attn_case([17, 64, 100, 256], Hh, d, L, 1 / 256, False, seed=5)
    got, st = _run_attn(off, ts, q, k, v, rp, rt, Hh, d, L, 1 / 256, False)
    assert st == 0
    T = int(off[-1])
    exp = O.pointwise_attention_fwd(q.reshape(T, Hh, d), k.reshape(T, Hh, d), v.reshape(T, Hh, d), off, ts, rp, rt,
                                    1 / 256, L, THR).reshape(T, Hh * d)
    assert_close(got, exp, *F32_TOL, what="O f32")


@pytest.mark.parametrize("o_bf16", [False, True])
def test_norm_gate_bf16(o_bf16):
    rng = np.random.default_rng(4)
    T, D = 257, 512
    o = 0.05 * rng.standard_normal((T, D)) + 0.02
    o = _bf16(o) if o_bf16 else o.astype(np.float32)
    udt = torch.bfloat16 if o_bf16 else torch.float16
    uvqk = _silu_like(rng, (T, 4 * D)) if o_bf16 else _f16(_silu_like(rng, (T, 4 * D)))
    gamma = (1 + 0.2 * rng.standard_normal(D)).astype(np.float32)
    beta = (0.2 * rng.standard_normal(D)).astype(np.float32)
    g = torch.empty(T, D, dtype=torch.bfloat16, device="cuda")
    mu = torch.empty(T, dtype=torch.float32, device="cuda")
    rstd = torch.empty(T, dtype=torch.float32, device="cuda")
    H.hstu_norm_gate_fwd(T, D, H.HSTU_BF16 if o_bf16 else H.HSTU_F32, H._dtype_code(torch.empty(0, dtype=udt)),
                         H.HSTU_BF16, to_dev(o, torch.bfloat16 if o_bf16 else torch.float32), D, to_dev(uvqk, udt),
                         4 * D,
                         to_dev(gamma, torch.float32), to_dev(beta, torch.float32), 1e-5, g, mu, rstd)
    ge, mue, rse = O.norm_gate_fwd(o, uvqk[:, :D], gamma, beta)
    assert_close(g.float().cpu().numpy(), ge, *BF16_TOL, what="G")
    assert_close(mu.cpu().numpy(), mue, 1e-6, 1e-5, what="mu")
    assert_close(rstd.cpu().numpy(), rse, 1e-6, 1e-4, what="rstd")


@pytest.mark.parametrize("xdt,ydt,gdt", [("bf16", "bf16", "bf16"), ("f32", "f32", "bf16"), ("bf16", "f32", "f16"),
                                         ("f32", "f32", "f16")])
def test_out_proj_bf16(xdt, ydt, gdt):
    rng = np.random.default_rng(6)
    T, D = 300, 512
    tg = torch.bfloat16 if gdt == "bf16" else torch.float16
    g = _bf16(rng.standard_normal((T, D))) if gdt == "bf16" else \
        rng.standard_normal((T, D)).astype(np.float16).astype(np.float32)
    W2 = _bf16(rng.standard_normal((D, D)) / np.sqrt(D))
    b2 = (0.1 * rng.standard_normal(D)).astype(np.float32)
    x = _bf16(rng.standard_normal((T, D))) if xdt == "bf16" else rng.standard_normal((T, D)).astype(np.float32)
    tx = torch.bfloat16 if xdt == "bf16" else torch.float32
    ty = torch.bfloat16 if ydt == "bf16" else torch.float32
    y = torch.empty(T, D, dtype=ty, device="cuda")
    y2 = torch.empty(T, D, dtype=torch.float16, device="cuda")
    gcode = H._dtype_code(y.new_empty(0, dtype=tg))
    ws = workspace(H.hstu_out_proj_workspace_size(D, gcode))
    H.hstu_out_proj_fwd(T, D, H.HSTU_BF16, gcode, to_dev(g, tg), to_dev(W2, torch.bfloat16),
                        to_dev(b2, torch.float32), to_dev(x, tx), H._dtype_code(y.new_empty(0, dtype=tx)), y,
                        H._dtype_code(y), y2, ws)
    ye = O.out_proj_fwd(g, W2, b2, x)
    tol = BF16_TOL if ydt == "bf16" else (1e-3, 1e-3)     # fp32 output: only accumulation-order error
    assert_close(y.float().cpu().numpy(), ye, *tol, what="Y")
    assert_close(y2.float().cpu().numpy(), ye, *BF16_TOL, what="Y fp16 copy")


# ---------------------------------------------------------------------------------------------
# whole layer
# ---------------------------------------------------------------------------------------------

def _run_layer(wl, x_dtype=None, y_dtype=None, x_override=None):
    bf = wl.dtype == "bf16"
    cdt = torch.bfloat16 if bf else torch.float32
    x_dtype = x_dtype or cdt
    y_dtype = y_dtype or cdt
    jag = JaggedBatch(wl.offsets, wl.timestamps, max_len=max(wl.max_len, 1))
    layer = DeviceLayer.upload(wl.layers[0], wl.D, wl.H, bf)
    run = LayerRunner(layer, jag, 1.0 / wl.N, wl.pos_max_len, x_dtype, y_dtype, keep_z=True)
    x = wl.x if x_override is None else x_override
    y = run.forward(to_dev(x, x_dtype))
    torch.cuda.synchronize()
    return y.float().cpu().numpy(), run


def test_layer_fwd_single_layer_fp32_workload():
    wl = W.make_workload("c1", seed=0)
    y, run = _run_layer(wl)
    assert run.device_status() == 0
    ye, _ = layer_oracle(wl)
    assert_close(y, ye, *F32_TOL, what="Y c1 fp32")


def test_layer_fwd_bf16_32_sequences_full():
    wl = W.make_workload("c2", seed=0)
    y, run = _run_layer(wl)
    assert run.device_status() == 0
    ye, inter = layer_oracle(wl)
    assert_close(y, ye, *BF16_TOL, what="Y c2 bf16")


def test_layer_fwd_long_sequences_every_row():
    """The long-sequence workload (8 Pareto-length sequences, T = 5759, d_model 512, H 8): all
    5759 x 512 outputs against the oracle."""
    wl = W.make_workload("c3", seed=0)
    y, run = _run_layer(wl)
    assert run.device_status() == 0
    ye, _ = layer_oracle(wl)
    assert y.shape == ye.shape == (wl.T, wl.D)
    assert_close(y, ye, *BF16_TOL, what="Y c3 bf16 (every row)")


def test_layer_fwd_fp32_residual_stream():
    """An fp32 residual stream: the oracle takes the fp32 X as it is (the kernels' fp16 f1 operand
    is their own rounding), the residual is added in fp32."""
    wl = W.make_workload("c4", seed=1, lengths=[200, 1, 0, 385, 128], layers=1)
    x32 = np.random.default_rng(9).standard_normal((wl.T, wl.D)).astype(np.float32)
    y, run = _run_layer(wl, torch.float32, torch.float32, x_override=x32)
    assert run.device_status() == 0
    ye, _ = layer_oracle(wl, x=x32)
    assert_close(y, ye, *BF16_TOL, what="Y fp32 residual")


def test_layer_fwd_fp16_copies_match_the_fp32_path():
    """x_f16 / y_f16: a layer fed the fp16 copy of its input gives the same bits as one that converts
    it itself, and its y_f16 output is the fp16 rounding of y."""
    wl = W.make_workload("c4", seed=3, lengths=[130, 77], layers=1)
    x32 = np.random.default_rng(4).standard_normal((wl.T, wl.D)).astype(np.float32)
    jag = JaggedBatch(wl.offsets, wl.timestamps)
    layer = DeviceLayer.upload(wl.layers[0], wl.D, wl.H, True)
    run = LayerRunner(layer, jag, 1.0 / wl.N, wl.pos_max_len, torch.float32, torch.float32, keep_z=True)
    x = to_dev(x32, torch.float32)
    y_a = run.forward(x).clone()
    y16 = torch.empty(wl.T, wl.D, dtype=torch.float16, device="cuda")
    y_b = run.forward(x, x.half(), y16).clone()
    torch.cuda.synchronize()
    assert run.device_status() == 0
    assert torch.equal(y_a, y_b)
    assert torch.equal(y16, y_b.half())


# ---------------------------------------------------------------------------------------------
# failure paths (host-injected; no GPU fault)
# ---------------------------------------------------------------------------------------------

def test_timeout_probe_reports_timeout_status():
    ws = workspace(256)
    H.hstu_set_wait_limit(1 << 20)
    try:
        H.hstu_debug_timeout_probe(ws)
        assert H.hstu_sync_status(ws) == 5
        assert H.hstu_sync_status(ws) == 0     # read resets it
    finally:
        H.hstu_set_wait_limit(0)


def test_offsets_violating_max_len_are_reported_not_read():
    off = W.offsets_from_lengths([10, 300])
    ts = np.zeros(310, np.int64)
    Hh, d = 1, 64
    q = np.zeros((310, 64), np.float32)
    got, st = _run_attn(off, ts, q, q, q, np.zeros(15, np.float32), np.zeros(128, np.float32), Hh, d, 8, 1.0, True,
                        max_len=100)
    assert st == 6
    assert np.all(np.isnan(got))           # nothing written


def test_empty_sequences_only():
    off = W.offsets_from_lengths([0, 0, 0])
    got, st = _run_attn(off, np.zeros(0, np.int64), np.zeros((0, 64)), np.zeros((0, 64)), np.zeros((0, 64)),
                        np.zeros(15, np.float32), np.zeros(128, np.float32), 1, 64, 8, 1.0, True, max_len=1)
    assert st == 0 and got.shape == (0, 64)


def test_profile_events_time_the_attention_kernel():
    """The timing hook records its two events around the attention forward kernel only: the kernel's
    time is positive and shorter than the whole call (work list and bias tiles included)."""
    wl = W.make_workload("c2", seed=0)
    Hh, d, L = wl.H, wl.D // wl.H, wl.pos_max_len
    off, ts, q, k, v, rp, rt = _attn_case(list(np.diff(wl.offsets)), Hh, d, L, 1 / wl.N, True, seed=3, f16=True)
    jag = JaggedBatch(off, ts)
    desc = H.make_attn_desc(Hh, d, d, 1 / wl.N, L, H.HSTU_F16, Hh * d, Hh * d, Hh * d, Hh * d)
    ws = workspace(H.hstu_attn_workspace_size(desc, jag.struct))
    out = torch.empty(jag.T, Hh * d, dtype=torch.float32, device="cuda")
    args = [to_dev(a, torch.float16) for a in (q, k, v)] + [to_dev(rp, torch.float32), to_dev(rt, torch.float32)]
    k0, k1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    H.hstu_profile_events(H.PROFILE_ATTN_FWD, k0, k1)
    try:
        for _ in range(3):
            c0.record()
            H.hstu_attn_fwd(desc, jag.struct, *args, out, ws)
            c1.record()
        torch.cuda.synchronize()
    finally:
        H.hstu_profile_events(H.PROFILE_ATTN_FWD)
    assert H.hstu_sync_status(ws) == 0
    kern, whole = k0.elapsed_time(k1), c0.elapsed_time(c1)
    assert 0 < kern < whole, (kern, whole)


@pytest.mark.parametrize("lengths", [
    [17, 64, 3, 1, 0, 40, 60, 5, 12, 64, 64, 1, 33, 130, 2],                 # one-warp work list (B <= 32)
    [(7 * i) % 66 for i in range(45)] + [200, 3],                              # block work list (B > 32)
])
def test_attn_fwd_packed_short_sequences(lengths):
    """Runs of short sequences (at most 64 tokens each, at most 128 rows together) share one 128-row
    tile, every row seeing only its own sequence's keys: the output must be the oracle's, with
    sequences of length 0 and 1 inside packs, packs that end exactly at 128 rows and long sequences
    between them."""
    Hh, d, L, inv_N = 2, 64, 300, 1.0 / 128
    off, ts, q, k, v, rp, rt = _attn_case(lengths, Hh, d, L, inv_N, True, seed=8, spread_ts=True, f16=True)
    got, st = _run_attn(off, ts, q, k, v, rp, rt, Hh, d, L, inv_N, True, f16=True)
    assert st == 0
    T = int(off[-1])
    exp = O.pointwise_attention_fwd(q.reshape(T, Hh, d), k.reshape(T, Hh, d), v.reshape(T, Hh, d), off, ts, rp, rt,
                                    inv_N, L, THR).reshape(T, Hh * d)
    scale = float(np.sqrt(np.mean(exp ** 2)))
    assert_close(got, exp, 1e-2 * scale, 1e-2, what="O (packed short sequences)")
