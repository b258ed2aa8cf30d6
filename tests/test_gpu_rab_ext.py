"""GPU parity of the richer relative bias (hstu_attn_fwd_ext / hstu_attn_bwd_ext): per-head rab_pos
and rab_time tables and the token-type term rab_type[type_i][type_j] ("HSTU: The First Exploration of
the Scaling Law", 7.1.4 Innovation 2, read as a sum of three looked-up terms), through the C ABI,
against the oracle's pointwise_attention_fwd_ext / _bwd_ext on ragged jagged batches.

Bound, as for the attention alone: |d| <= 1e-2 rms(ref) + 1e-2 |ref| per tensor (16-bit operands,
fp32 accumulation). A token type outside [0, n_types) is reported as HSTU_ERR_DEVICE.
"""
import numpy as np
import pytest
import torch

from oracle import hstu_oracle as O
from hstu_sequential_transduction_causal_b200 import hstu as H
from hstu_sequential_transduction_causal_b200.runtime import JaggedBatch, to_dev, workspace
from tests._util import THR, assert_close
from tests.test_gpu_forward import _attn_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from hstu_sequential_transduction_causal_b200 import build
    build.build()
    H.lib()
    torch.cuda.init()


def _case(lengths, Hh, L, per_head, n_types, seed, spread=True):
    d = 64
    off, ts, q, k, v, rp, rt = _attn_case(lengths, Hh, d, L, 1.0, True, seed=seed, spread_ts=spread, f16=True)
    rng = np.random.default_rng(seed + 50)
    T = int(off[-1])
    hb = Hh if per_head else 1
    rp = rng.standard_normal((hb, 2 * L - 1)).astype(np.float32)
    rt = rng.standard_normal((hb, 128)).astype(np.float32)
    types = rng.integers(0, max(n_types, 1), T).astype(np.int32)
    ty = rng.standard_normal((hb, max(n_types, 1), max(n_types, 1))).astype(np.float32)
    if not per_head:
        rp, rt, ty = rp[0], rt[0], ty[0]
    return off, ts, q, k, v, rp, rt, types, ty


def _oracle_tables(per_head, n_types, rp, rt, ty, types):
    return dict(token_type=types if n_types else None, rab_type=ty if n_types else None, per_head=per_head)


@pytest.mark.parametrize("per_head,n_types", [(True, 0), (True, 3), (False, 5), (False, 1)])
def test_attn_fwd_ext(per_head, n_types):
    lengths = [1, 127, 128, 129, 300, 0, 513, 64]
    Hh, d, L, inv_N = 2, 64, 600, 1.0 / 512
    off, ts, q, k, v, rp, rt, types, ty = _case(lengths, Hh, L, per_head, n_types, seed=21)
    T = int(off[-1])
    jag = JaggedBatch(off, ts)
    desc = H.make_attn_desc(Hh, d, d, inv_N, L, H.HSTU_F16, Hh * d, Hh * d, Hh * d, Hh * d)
    dty, dtt = to_dev(types, torch.int32), to_dev(ty, torch.float32)
    ext = H.make_rab_ext(per_head, n_types, dty if n_types else None, dtt if n_types else None)
    ws = workspace(H.hstu_attn_ext_workspace_size(desc, jag.struct, ext))
    out = torch.full((T, Hh * d), float("nan"), dtype=torch.float32, device="cuda")
    H.hstu_attn_fwd_ext(desc, jag.struct, ext, to_dev(q, torch.float16), to_dev(k, torch.float16),
                        to_dev(v, torch.float16), to_dev(rp, torch.float32), to_dev(rt, torch.float32), out, ws)
    torch.cuda.synchronize()
    assert H.hstu_sync_status(ws) == 0
    exp = O.pointwise_attention_fwd_ext(q.reshape(T, Hh, d), k.reshape(T, Hh, d), v.reshape(T, Hh, d), off, ts, rp,
                                        rt, inv_N, L, THR, **_oracle_tables(per_head, n_types, rp, rt, ty, types))
    exp = exp.reshape(T, Hh * d)
    scale = float(np.sqrt(np.mean(exp ** 2)))
    assert_close(out.cpu().numpy(), exp, 1e-2 * scale, 1e-2, what=f"O ext per_head={per_head} n_types={n_types}")


@pytest.mark.parametrize("per_head,n_types", [(True, 3), (False, 4), (True, 0)])
def test_attn_bwd_ext(per_head, n_types):
    lengths = [1, 127, 128, 129, 300, 0, 260]
    Hh, d, L, inv_N = 2, 64, 400, 1.0 / 512
    off, ts, q, k, v, rp, rt, types, ty = _case(lengths, Hh, L, per_head, n_types, seed=33)
    T = int(off[-1])
    rng = np.random.default_rng(7)
    do = rng.standard_normal((T, Hh * d)).astype(np.float16).astype(np.float32)
    jag = JaggedBatch(off, ts)
    desc = H.make_attn_desc(Hh, d, d, inv_N, L, H.HSTU_F16, Hh * d, Hh * d, Hh * d, Hh * d)
    dty, dtt = to_dev(types, torch.int32), to_dev(ty, torch.float32)
    ext = H.make_rab_ext(per_head, n_types, dty if n_types else None, dtt if n_types else None)
    ws = workspace(H.hstu_attn_bwd_ext_workspace_size(desc, jag.struct, ext))
    outs = [torch.full((T, Hh * d), float("nan"), dtype=torch.float32, device="cuda") for _ in range(3)]
    drp = torch.full(rp.shape, float("nan"), dtype=torch.float32, device="cuda")
    drt = torch.full(rt.shape, float("nan"), dtype=torch.float32, device="cuda")
    drty = torch.full(ty.shape, float("nan"), dtype=torch.float32, device="cuda") if n_types else None
    f16 = torch.float16
    H.hstu_attn_bwd_ext(desc, jag.struct, ext, to_dev(q, f16), to_dev(k, f16), to_dev(v, f16), to_dev(do, f16),
                        to_dev(rp, torch.float32), to_dev(rt, torch.float32), *outs, drp, drt, drty, ws)
    torch.cuda.synchronize()
    assert H.hstu_sync_status(ws) == 0
    exp = O.pointwise_attention_bwd_ext(q.reshape(T, Hh, d), k.reshape(T, Hh, d), v.reshape(T, Hh, d),
                                        do.reshape(T, Hh, d), off, ts, rp, rt, inv_N, L, THR,
                                        **_oracle_tables(per_head, n_types, rp, rt, ty, types))
    got = [t.cpu().numpy() for t in outs] + [drp.cpu().numpy(), drt.cpu().numpy()]
    want = [e.reshape(T, Hh * d) for e in exp[:3]] + [exp[3], exp[4]]
    names = ["dq", "dk", "dv", "drab_pos", "drab_time"]
    if n_types:
        got.append(drty.cpu().numpy())
        want.append(exp[5])
        names.append("drab_type")
    for g, e, name in zip(got, want, names):
        scale = float(np.sqrt(np.mean(e ** 2))) if e.size else 0.0
        assert_close(g, e, 1e-2 * scale + 1e-12, 1e-2, what=f"{name} per_head={per_head} n_types={n_types}")


def test_attn_fwd_ext_reports_out_of_range_types():
    lengths = [130, 7]
    Hh, d, L = 2, 64, 200
    off, ts, q, k, v, rp, rt, types, ty = _case(lengths, Hh, L, False, 3, seed=5)
    types[40] = 3           # one past the last type
    T = int(off[-1])
    jag = JaggedBatch(off, ts)
    desc = H.make_attn_desc(Hh, d, d, 1.0 / 256, L, H.HSTU_F16, Hh * d, Hh * d, Hh * d, Hh * d)
    dty, dtt = to_dev(types, torch.int32), to_dev(ty, torch.float32)   # kept alive: ext holds pointers
    ext = H.make_rab_ext(False, 3, dty, dtt)
    ws = workspace(H.hstu_attn_ext_workspace_size(desc, jag.struct, ext))
    out = torch.empty((T, Hh * d), dtype=torch.float32, device="cuda")
    H.hstu_attn_fwd_ext(desc, jag.struct, ext, to_dev(q, torch.float16), to_dev(k, torch.float16),
                        to_dev(v, torch.float16), to_dev(rp, torch.float32), to_dev(rt, torch.float32), out, ws)
    torch.cuda.synchronize()
    assert H.hstu_sync_status(ws) == 6
