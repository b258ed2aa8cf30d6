"""The attention forward for callers that cannot allocate device memory.

Such callers (a serving process whose whole memory budget is reserved at start-up, a plain C host
without a device allocator) cannot pass a workspace, so ``hstu_attn_fwd_noalloc`` keeps its scratch
in a fixed array inside the library. This file checks, through the C ABI:
  - on two different batches called back to back (the second call must not see the first call's
    work list), that the output matches the CPU oracle within the attention's bound and the
    workspace entry point's output, and that the call's own status word (read with
    ``hstu_attn_fwd_noalloc_status``) is clear;
  - that offsets violating the jagged contract are reported through that status word, with
    nothing written.
Refusal of batches too large for the fixed array is checked on the CPU (test_abi_validation.py),
where no kernel could ever be reached. Named so pytest collects it last.
"""
import numpy as np
import pytest
import torch

from oracle import hstu_oracle as O
from hstu_sequential_transduction_causal_b200 import hstu as H
from hstu_sequential_transduction_causal_b200 import workloads as W
from hstu_sequential_transduction_causal_b200.runtime import JaggedBatch, to_dev, workspace
from tests._util import THR, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from hstu_sequential_transduction_causal_b200 import build
    build.build()
    H.lib()
    torch.cuda.init()


def _batch(lengths, seed, Hh=2, d=64, L=1100, inv_N=1.0 / 1024):
    rng = np.random.default_rng(seed)
    off = W.offsets_from_lengths(lengths)
    T = int(off[-1])
    ts = W.draw_timestamps(rng, lengths)
    z = rng.standard_normal((3, T, Hh * d))
    qkv = [(z[i] / (1 + np.exp(-z[i]))).astype(np.float16).astype(np.float64) for i in range(3)]
    rp = rng.standard_normal(2 * L - 1).astype(np.float32)
    rt = rng.standard_normal(128).astype(np.float32)
    jag = JaggedBatch(off, ts)
    desc = H.make_attn_desc(Hh, d, d, inv_N, L, H.HSTU_F16, Hh * d, Hh * d, Hh * d, Hh * d)
    exp = O.pointwise_attention_fwd(*(a.reshape(T, Hh, d) for a in qkv), off, ts, rp, rt, inv_N, L,
                                    THR).reshape(T, Hh * d)
    dev = [to_dev(a, torch.float16) for a in qkv] + [to_dev(rp, torch.float32), to_dev(rt, torch.float32)]
    return jag, desc, dev, exp


def test_noalloc_matches_oracle_and_workspace_entry_point_on_two_calls_in_a_row():
    for lengths, seed in (([300, 1, 0, 129, 1024, 64], 0), ([5, 700, 128], 1)):
        jag, desc, (q, k, v, rp, rt), exp = _batch(lengths, seed)
        T, C = jag.T, q.shape[1]
        got = torch.full((T, C), float("nan"), dtype=torch.float32, device="cuda")
        H.hstu_attn_fwd_noalloc(desc, jag.struct, q, k, v, rp, rt, got)
        assert H.hstu_attn_fwd_noalloc_status() == 0
        ref = torch.full((T, C), float("nan"), dtype=torch.float32, device="cuda")
        ws = workspace(H.hstu_attn_workspace_size(desc, jag.struct))
        H.hstu_attn_fwd(desc, jag.struct, q, k, v, rp, rt, ref, ws)
        torch.cuda.synchronize()
        assert H.hstu_sync_status(ws) == 0
        g, r = got.cpu().numpy(), ref.cpu().numpy()
        scale = float(np.sqrt(np.mean(exp ** 2)))
        # the attention output alone: |d| <= 1e-2 rms(ref) + 1e-2 |ref| (16-bit operands, fp32 accumulate)
        assert_close(g, exp, 1e-2 * scale, 1e-2, what=f"noalloc O vs oracle (seed {seed})")
        assert_close(g, r, 1e-2 * scale, 1e-2, what=f"noalloc O vs workspace entry point (seed {seed})")


def test_noalloc_reports_offsets_violating_max_len():
    """A sequence longer than max_len (host-injected contract violation): the work list is emptied,
    nothing is written, and the status word of the built-in scratch says HSTU_ERR_DEVICE; the next
    good call starts from a clear status again."""
    off = W.offsets_from_lengths([10, 300])
    jag = JaggedBatch(off, np.zeros(310, np.int64), max_len=100)
    desc = H.make_attn_desc(1, 64, 64, 1.0, 8, H.HSTU_F16, 64, 64, 64, 64)
    z = torch.zeros(310, 64, dtype=torch.float16, device="cuda")
    tables = (torch.zeros(15, device="cuda"), torch.zeros(128, device="cuda"))
    out = torch.full((310, 64), float("nan"), dtype=torch.float32, device="cuda")
    H.hstu_attn_fwd_noalloc(desc, jag.struct, z, z, z, *tables, out)
    assert H.hstu_attn_fwd_noalloc_status() == 6
    assert torch.isnan(out).all()
    good = JaggedBatch(off, np.zeros(310, np.int64))
    H.hstu_attn_fwd_noalloc(desc, good.struct, z, z, z, *tables, out)
    assert H.hstu_attn_fwd_noalloc_status() == 0
    assert torch.isfinite(out).all()
