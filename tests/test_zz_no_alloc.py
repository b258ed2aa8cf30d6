"""The attention forward for callers that cannot allocate device memory.

Such callers (a serving process whose whole memory budget is reserved at start-up, a plain C host
without a device allocator) cannot pass a workspace, so ``hstu_attn_fwd_noalloc`` keeps its scratch
in a fixed array inside the library. This file checks, through the C ABI, that it returns what the
workspace entry point returns, on two different batches called back to back (the second call must
not see the first call's work list), and that a batch too large for the fixed array is refused
before anything runs. Named so pytest collects it last.
"""
import numpy as np
import pytest
import torch

from hstu_sequential_transduction_causal_b200 import hstu as H
from hstu_sequential_transduction_causal_b200 import workloads as W
from hstu_sequential_transduction_causal_b200.runtime import JaggedBatch, to_dev, workspace

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from hstu_sequential_transduction_causal_b200 import build
    build.build()
    H.lib()
    torch.cuda.init()


def _batch(lengths, seed, Hh=2, d=64, L=1100):
    rng = np.random.default_rng(seed)
    off = W.offsets_from_lengths(lengths)
    T = int(off[-1])
    ts = W.draw_timestamps(rng, lengths)
    z = rng.standard_normal((3, T, Hh * d))
    qkv = [to_dev(z[i] / (1 + np.exp(-z[i])), torch.float16) for i in range(3)]
    rp = to_dev(rng.standard_normal(2 * L - 1), torch.float32)
    rt = to_dev(rng.standard_normal(128), torch.float32)
    jag = JaggedBatch(off, ts)
    desc = H.make_attn_desc(Hh, d, d, 1.0 / 1024, L, H.HSTU_F16, Hh * d, Hh * d, Hh * d, Hh * d)
    return jag, desc, qkv, rp, rt


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    for lengths, seed in (([300, 1, 0, 129, 1024, 64], 0), ([5, 700, 128], 1)):
        jag, desc, (q, k, v), rp, rt = _batch(lengths, seed)
        T, C = jag.T, q.shape[1]
        ref = torch.full((T, C), float("nan"), dtype=torch.float32, device="cuda")
        ws = workspace(H.hstu_attn_workspace_size(desc, jag.struct))
        H.hstu_attn_fwd(desc, jag.struct, q, k, v, rp, rt, ref, ws)
        got = torch.full((T, C), float("nan"), dtype=torch.float32, device="cuda")
        H.hstu_attn_fwd_noalloc(desc, jag.struct, q, k, v, rp, rt, got)
        torch.cuda.synchronize()
        assert H.hstu_sync_status(ws) == 0
        r, g = ref.cpu().numpy(), got.cpu().numpy()
        assert np.all(np.isfinite(g))
        scale = float(np.sqrt(np.mean(r ** 2)))
        err = np.abs(g - r)
        assert np.all(err <= 1e-2 * scale + 1e-2 * np.abs(r)), float(err.max())


def test_noalloc_refuses_batches_beyond_its_fixed_scratch():
    # one sequence of 70,000 tiles: more work items than HSTU_NOALLOC_MAX_ITEMS; the pointers are
    # never dereferenced because the size check comes first
    jag = H.hstu_jagged_t(B=1, max_len=1 << 30, T=128 * 70000, offsets=256, timestamps=256)
    desc = H.make_attn_desc(2, 64, 64, 1.0, 8, H.HSTU_F16, 128, 128, 128, 128)
    code = H.lib().hstu_attn_fwd_noalloc(desc, jag, 256, 256, 256, 256, 256, 256, None)
    assert code == 3     # HSTU_ERR_WORKSPACE, nothing enqueued
