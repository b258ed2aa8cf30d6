"""GPU parity of M-FALCON candidate scoring (hstu_falcon_fwd) against the oracle.

The residual stream between the stacked layers is fp32, so the oracle (fp64 throughout) is compared
with no rounding between layers. Checks: ragged prefixes including an empty and a one-token prefix, a candidate count that is not a
multiple of the 128-row tile, micro-batch sizes b_m in {m, 2, 1} (the result must not depend on b_m:
bit-identical on the GPU), reuse of a cache built by an earlier call (cache_valid = 1, bit-identical),
the prefix's own last-layer output, and the full 16 x 2048-prefix, 1024-candidate, 4-layer ranking
workload on sampled users and candidates.
"""
import numpy as np
import pytest
import torch

from oracle import hstu_oracle as O
from hstu_sequential_transduction_causal_b200 import hstu as H
from hstu_sequential_transduction_causal_b200 import workloads as W
from hstu_sequential_transduction_causal_b200.runtime import DeviceLayer, JaggedBatch, to_dev, workspace
from tests._util import BF16_TOL, THR, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from hstu_sequential_transduction_causal_b200 import build
    build.build()
    H.lib()
    torch.cuda.init()


class FalconRun:
    """Device buffers of one M-FALCON problem; run() calls hstu_falcon_fwd."""

    def __init__(self, fw, b_m):
        self.fw = fw
        D, L = fw.D, len(fw.layers)
        lens = np.diff(fw.prefix_offsets)
        self.jag = JaggedBatch(fw.prefix_offsets, fw.prefix_ts, max_len=int(lens.max()) if lens.size else 0)
        self.layers = [DeviceLayer.upload(p, D, fw.H, True) for p in fw.layers]
        self.weights = [lay.weights() for lay in self.layers]
        self.desc = H.make_falcon_desc(L, fw.users, fw.m, b_m, D, fw.H, 1.0 / fw.N, fw.pos_max_len)
        self.px = to_dev(fw.prefix_x, torch.bfloat16)
        self.cx = to_dev(fw.cand_x, torch.bfloat16)
        self.req = to_dev(fw.request_ts, torch.int64)
        nbytes = H.hstu_falcon_cache_size(self.desc, self.jag.struct)
        self.cache = torch.full((max(nbytes, 2) // 2,), float("nan"), dtype=torch.float16, device="cuda")
        self.ws = workspace(H.hstu_falcon_workspace_size(self.desc, self.jag.struct))
        self.prefix_out = torch.full((max(self.jag.T, 1), D), float("nan"), dtype=torch.float32, device="cuda")

    def run(self, cache_valid=0):
        out = torch.full((self.fw.users * self.fw.m, self.fw.D), float("nan"), dtype=torch.float32, device="cuda")
        H.hstu_falcon_fwd(self.desc, self.weights, self.jag.struct, self.px, self.cache, cache_valid,
                          self.prefix_out, self.cx, self.req, out, self.ws)
        torch.cuda.synchronize()
        assert H.hstu_sync_status(self.ws) == 0
        return out.float().cpu().numpy()


def _oracle(fw):
    return O.falcon_fwd(fw.layers, fw.prefix_offsets, fw.prefix_ts, fw.prefix_x, fw.cand_x, fw.request_ts,
                        fw.m, fw.H, 1.0 / fw.N, fw.pos_max_len, THR)


def test_falcon_ragged_prefixes_and_micro_batches():
    fw = W.make_falcon_workload(seed=11, prefix_lengths=[130, 0, 1, 257], m=5, b_m=2, D=128, H=2, layers=2,
                                N=300, pos_max_len=300)
    yc_ref, yp_ref = _oracle(fw)
    runs = {}
    for b_m in (fw.m, 2, 1):
        r = FalconRun(fw, b_m)
        runs[b_m] = r.run()
        assert_close(runs[b_m], yc_ref, *BF16_TOL, what=f"candidates b_m={b_m}")
        assert_close(r.prefix_out.float().cpu().numpy(), yp_ref, *BF16_TOL, what="prefix output")
    # one kernel sequence per candidate row whatever the micro-batch: identical bits
    assert np.array_equal(runs[fw.m], runs[2]) and np.array_equal(runs[fw.m], runs[1])


def test_falcon_cache_reuse_is_identical():
    fw = W.make_falcon_workload(seed=12, prefix_lengths=[200, 64, 129], m=130, b_m=64, D=128, H=2, layers=2,
                                N=300, pos_max_len=300)
    r = FalconRun(fw, fw.b_m)
    first = r.run(cache_valid=0)
    yc_ref, _ = _oracle(fw)
    assert_close(first, yc_ref, *BF16_TOL, what="candidates (cache built)")
    # a second call on the cached K, V: prefix_x is not read, so poison it first
    r.px.fill_(float("nan"))
    second = r.run(cache_valid=1)
    assert np.array_equal(first, second)


def test_falcon_ranking_workload_every_candidate():
    """16 users x 2048-token prefixes, 1024 candidates per user in micro-batches of 256, 4 layers,
    d_model 512, H 8: every one of the 16384 candidate outputs (and the prefix's last-layer
    output) against the oracle, which needs about two minutes of host time."""
    fw = W.make_falcon_workload(seed=0)
    r = FalconRun(fw, fw.b_m)
    got = r.run()
    assert np.all(np.isfinite(got))
    yc_ref, yp_ref = _oracle(fw)
    assert got.shape == yc_ref.shape == (16 * 1024, fw.D)
    assert_close(got, yc_ref, *BF16_TOL, what="ranking workload candidates (all)")
    assert_close(r.prefix_out.float().cpu().numpy(), yp_ref, *BF16_TOL, what="ranking workload prefix output")


def test_falcon_prefix_append_matches_a_rebuilt_prefix():
    """hstu_falcon_append grows cached prefixes of 130, 0, 1 and 257 tokens by 5, 3, 0 and 130 new
    actions. The combined cache must be bit-identical to one built from scratch over the combined
    prefixes (each row's K, V come from the same per-row arithmetic), the appended tokens' output
    must equal the rows a full causal forward over the combined prefixes gives them (bit-identical
    on the GPU, and within the bf16 bound of the oracle), and candidates scored from the appended
    cache must match the oracle's M-FALCON over the combined prefixes."""
    old_lens, app_lens = [130, 0, 1, 257], [5, 3, 0, 130]
    fw = W.make_falcon_workload(seed=14, prefix_lengths=[o + a for o, a in zip(old_lens, app_lens)], m=7, b_m=7,
                                D=128, H=2, layers=2, N=400, pos_max_len=400)
    off = fw.prefix_offsets
    rows_old = np.concatenate([np.arange(off[u], off[u] + old_lens[u]) for u in range(4)]).astype(np.int64)
    rows_app = np.concatenate([np.arange(off[u] + old_lens[u], off[u + 1]) for u in range(4)]).astype(np.int64)
    fw_old = W.FalconWorkload(D=fw.D, H=fw.H, N=fw.N, pos_max_len=fw.pos_max_len, layers=fw.layers,
                              prefix_offsets=W.offsets_from_lengths(old_lens), prefix_ts=fw.prefix_ts[rows_old],
                              prefix_x=fw.prefix_x[rows_old], cand_x=fw.cand_x, request_ts=fw.request_ts, m=fw.m,
                              b_m=fw.b_m)
    r_old = FalconRun(fw_old, fw.b_m)
    r_old.run(cache_valid=0)
    r_new = FalconRun(fw, fw.b_m)           # the combined prefixes, built from scratch
    r_new.run(cache_valid=0)
    jag_app = JaggedBatch(W.offsets_from_lengths(app_lens), fw.prefix_ts[rows_app], max_len=max(app_lens))
    cache = torch.full_like(r_new.cache, float("nan"))
    app_out = torch.full((len(rows_app), fw.D), float("nan"), dtype=torch.float32, device="cuda")
    ws = workspace(H.hstu_falcon_append_workspace_size(r_new.desc, r_old.jag.struct, jag_app.struct,
                                                       r_new.jag.struct))
    H.hstu_falcon_append(r_new.desc, r_new.weights, r_old.jag.struct, r_old.cache, jag_app.struct,
                         to_dev(fw.prefix_x[rows_app], torch.bfloat16), r_new.jag.struct, cache, app_out, ws)
    torch.cuda.synchronize()
    assert H.hstu_sync_status(ws) == 0
    assert torch.equal(cache, r_new.cache)
    assert torch.equal(app_out, r_new.prefix_out[torch.from_numpy(rows_app).cuda()])
    yc_ref, yp_ref = _oracle(fw)
    assert_close(app_out.cpu().numpy(), yp_ref[rows_app], *BF16_TOL, what="appended tokens' output")
    r_new.cache.copy_(cache)
    r_new.px.fill_(float("nan"))            # cache_valid = 1 does not read the prefix input
    assert_close(r_new.run(cache_valid=1), yc_ref, *BF16_TOL, what="candidates on the appended cache")


def test_falcon_append_of_nothing_keeps_the_cache():
    lens = [64, 0, 200]
    fw = W.make_falcon_workload(seed=15, prefix_lengths=lens, m=3, b_m=3, D=128, H=2, layers=2, N=300,
                                pos_max_len=300)
    r = FalconRun(fw, fw.b_m)
    r.run(cache_valid=0)
    jag_app = JaggedBatch(np.zeros(4, np.int64), np.zeros(0, np.int64), max_len=0)
    cache = torch.full_like(r.cache, float("nan"))
    ws = workspace(H.hstu_falcon_append_workspace_size(r.desc, r.jag.struct, jag_app.struct, r.jag.struct))
    H.hstu_falcon_append(r.desc, r.weights, r.jag.struct, r.cache, jag_app.struct, None, r.jag.struct, cache, None, ws)
    torch.cuda.synchronize()
    assert H.hstu_sync_status(ws) == 0
    assert torch.equal(cache, r.cache)
