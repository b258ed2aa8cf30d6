"""GPU parity of the attention backward and the layer backward against the oracle's closed-form
gradients (which are themselves pinned to finite differences in test_oracle_pins.py).

Tolerance per gradient tensor: |d| <= 1e-2 rms(ref) + 1e-2 |ref| for the attention alone (16-bit
operands, fp32 accumulation; the scale term keeps entries near zero from failing on rounding
of their large neighbours); the layer's final gradients use the bf16 bound |d| <= 1e-2 + 1e-2 |ref|.
"""
import numpy as np
import pytest
import torch

from oracle import hstu_oracle as O
from hstu_sequential_transduction_causal_b200 import hstu as H
from hstu_sequential_transduction_causal_b200.runtime import JaggedBatch, to_dev, workspace
from tests._util import THR, assert_close
from tests.test_gpu_forward import _attn_case, _f16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from hstu_sequential_transduction_causal_b200 import build
    build.build()
    H.lib()
    torch.cuda.init()


def _run_attn_bwd(lengths, Hh, L, inv_N, seed, spread=False, f16=True, do_scale=1.0):
    d = 64
    off, ts, q, k, v, rp, rt = _attn_case(lengths, Hh, d, L, inv_N, True, seed=seed, spread_ts=spread, f16=f16)
    T = int(off[-1])
    rng = np.random.default_rng(seed + 100)
    cast = _f16 if f16 else (lambda a: __import__("hstu_sequential_transduction_causal_b200.workloads",
                                                  fromlist=["round_bf16"]).round_bf16(a))
    do = cast(do_scale * rng.standard_normal((T, Hh * d)))
    tdt = torch.float16 if f16 else torch.bfloat16
    jag = JaggedBatch(off, ts)
    desc = H.make_attn_desc(Hh, d, d, inv_N, L, H.HSTU_F16 if f16 else H.HSTU_BF16, Hh * d, Hh * d, Hh * d, Hh * d)
    ws = workspace(H.hstu_attn_bwd_workspace_size(desc, jag.struct))
    outs = [torch.full((T, Hh * d), float("nan"), dtype=torch.float32, device="cuda") for _ in range(3)]
    drp = torch.full((2 * L - 1,), float("nan"), dtype=torch.float32, device="cuda")
    drt = torch.full((128,), float("nan"), dtype=torch.float32, device="cuda")
    H.hstu_attn_bwd(desc, jag.struct, to_dev(q, tdt), to_dev(k, tdt), to_dev(v, tdt), to_dev(do, tdt),
                    to_dev(rp, torch.float32), to_dev(rt, torch.float32), *outs, drp, drt, ws)
    torch.cuda.synchronize()
    st = H.hstu_sync_status(ws)
    got = [t.cpu().numpy() for t in outs] + [drp.cpu().numpy(), drt.cpu().numpy()]
    exp = O.pointwise_attention_bwd(q.reshape(T, Hh, d), k.reshape(T, Hh, d), v.reshape(T, Hh, d),
                                    do.reshape(T, Hh, d), off, ts, rp, rt, inv_N, L, THR)
    exp = [e.reshape(T, Hh * d) for e in exp[:3]] + list(exp[3:])
    return st, got, exp


def _check(got, exp, names=("dq", "dk", "dv", "drab_pos", "drab_time")):
    for g, e, name in zip(got, exp, names):
        scale = float(np.sqrt(np.mean(e ** 2))) if e.size else 0.0
        assert_close(g, e, 1e-2 * scale + 1e-12, 1e-2, what=name)


@pytest.mark.parametrize("spread", [False, True])
def test_attn_bwd_fp16_ragged(spread):
    st, got, exp = _run_attn_bwd([1, 127, 128, 129, 300, 0, 513, 64], 2, 600, 1.0 / 512, seed=3, spread=spread)
    assert st == 0
    _check(got, exp)


def test_attn_bwd_bf16_operands():
    st, got, exp = _run_attn_bwd([200, 5, 260], 2, 300, 1.0 / 256, seed=4, f16=False)
    assert st == 0
    _check(got, exp)


def test_attn_bwd_odd_heads_long_sequence():
    st, got, exp = _run_attn_bwd([1100, 3], 3, 1200, 1.0 / 2048, seed=5)
    assert st == 0
    _check(got, exp)


@pytest.mark.parametrize("lengths", [
    [17, 64, 3, 1, 0, 40, 60, 5, 12, 64, 64, 1, 33, 130, 2],
    [(7 * i) % 66 for i in range(45)] + [200, 3],
])
def test_attn_bwd_packed_short_sequences(lengths):
    """The backward over packs of short sequences (one key tile per pack, queries limited to the key's
    own sequence, the packed members' own pairs skipped by the table gradients)."""
    st, got, exp = _run_attn_bwd(lengths, 2, 300, 1.0 / 128, seed=9, spread=True)
    assert st == 0
    _check(got, exp)
