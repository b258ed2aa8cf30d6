"""Out-of-bounds writes, checked indices and the fp16 range, on the GPU.

compute-sanitizer is not available on this machine, so:
  - every output of the layer forward and backward (and of the standalone attention calls) sits
    between canary guard regions that must come back unchanged;
  - the checked-index build (build.py --debug, loaded under HSTU_DEBUG=1) runs a ragged layer
    forward + backward and the richer-bias attention in a child process: no check may fire, and
    the results still match the oracle;
  - values beyond the fp16 range in BF16 mode's fp16 intermediates are reported (HSTU_ERR_DEVICE)
    instead of passing as inf.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from oracle import hstu_oracle as O
from hstu_sequential_transduction_causal_b200 import hstu as H
from hstu_sequential_transduction_causal_b200 import workloads as W
from hstu_sequential_transduction_causal_b200.runtime import (DeviceLayer, JaggedBatch, SavedActs, to_dev,
                                                              workspace)
from tests._util import THR, assert_close, guarded

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from hstu_sequential_transduction_causal_b200 import build
    build.build()
    H.lib()
    torch.cuda.init()


def test_layer_forward_backward_outputs_keep_their_canaries():
    lengths = [1, 127, 0, 129, 300, 64, 513]
    wl = W.make_workload("c2", seed=3, lengths=lengths, D=256, H=4, N=600, pos_max_len=600, backward=True)
    T, D = wl.T, wl.D
    jag = JaggedBatch(wl.offsets, wl.timestamps)
    layer = DeviceLayer.upload(wl.layers[0], D, wl.H, True)
    desc = H.make_layer_desc(D, wl.H, 1.0 / wl.N, wl.pos_max_len, H.HSTU_BF16, H.HSTU_BF16, H.HSTU_BF16)
    checks = []

    def g(shape, dtype, fill=float("nan")):
        t, c = guarded(shape, dtype, fill)
        checks.append(c)
        return t

    sv = SavedActs(uvqk=g((T, 4 * D), torch.float16), z=g((T, 4 * D), torch.float16),
                   o=g((T, D), torch.float32), g=g((T, D), torch.float16), mu=g((T,), torch.float32),
                   rstd=g((T,), torch.float32))
    y = g((T, D), torch.bfloat16)
    x = to_dev(wl.x, torch.bfloat16)
    ws = workspace(max(H.hstu_layer_workspace_size(desc, jag.struct), H.hstu_layer_bwd_workspace_size(desc, jag.struct)))
    H.hstu_layer_fwd(desc, jag.struct, layer.weights(), x, None, y, None, sv.struct(), ws)
    grads = [g((n,), torch.float32, 0.0)
             for n in (4 * D * D, 4 * D, D * D, D, D, D, 2 * wl.pos_max_len - 1, 128)]
    dx = g((T, D), torch.bfloat16)
    H.hstu_layer_bwd(desc, jag.struct, layer.weights(), x, None, sv.struct(), to_dev(wl.dy, torch.bfloat16), None, dx,
                     None, H.layer_grads(*grads), ws)
    torch.cuda.synchronize()
    assert H.hstu_sync_status(ws) == 0
    names = ["uvqk", "z", "o", "g", "mu", "rstd", "y"] + [f"grad{i}" for i in range(8)] + ["dx"]
    for c, name in zip(checks, names):
        c(name)
    for t, name in ((y, "y"), (dx, "dx"), (sv.o, "o")):
        assert bool(torch.isfinite(t.float()).all()), f"{name}: an element was not written"


def test_attention_outputs_keep_their_canaries():
    lengths = [5, 128, 0, 257, 1, 700]
    rng = np.random.default_rng(4)
    off = W.offsets_from_lengths(lengths)
    T, Hh, d, L = int(off[-1]), 2, 64, 800
    ts = W.draw_timestamps(rng, lengths)
    z = rng.standard_normal((4, T, Hh * d))
    q, k, v, do = [(a / (1 + np.exp(-a))).astype(np.float16) for a in z]
    rp, rt = rng.standard_normal(2 * L - 1).astype(np.float32), rng.standard_normal(128).astype(np.float32)
    jag = JaggedBatch(off, ts)
    desc = H.make_attn_desc(Hh, d, d, 1.0 / 512, L, H.HSTU_F16, Hh * d, Hh * d, Hh * d, Hh * d)
    dev = [to_dev(a, torch.float16) for a in (q, k, v, do)] + [to_dev(rp, torch.float32), to_dev(rt, torch.float32)]
    out, c_out = guarded((T, Hh * d), torch.float32)
    ws = workspace(H.hstu_attn_bwd_workspace_size(desc, jag.struct))
    H.hstu_attn_fwd(desc, jag.struct, dev[0], dev[1], dev[2], dev[4], dev[5], out, ws)
    gr = [guarded((T, Hh * d), torch.float32, 0.0) for _ in range(3)]
    drp, c_drp = guarded((2 * L - 1,), torch.float32, 0.0)
    drt, c_drt = guarded((128,), torch.float32, 0.0)
    H.hstu_attn_bwd(desc, jag.struct, dev[0], dev[1], dev[2], dev[3], dev[4], dev[5], *[t for t, _ in gr], drp, drt,
                    ws)
    torch.cuda.synchronize()
    assert H.hstu_sync_status(ws) == 0
    c_out("O")
    for (t, c), name in zip(gr, ("dq", "dk", "dv")):
        c(name)
    c_drp("d rab_pos")
    c_drt("d rab_time")
    exp = O.pointwise_attention_fwd(*(a.astype(np.float64).reshape(T, Hh, d) for a in (q, k, v)), off, ts, rp, rt,
                                    1.0 / 512, L, THR).reshape(T, Hh * d)
    assert_close(out.cpu().numpy(), exp, 1e-2 * float(np.sqrt(np.mean(exp ** 2))), 1e-2, what="O")


_CHILD = r"""
import sys
import numpy as np, torch
sys.path.insert(0, sys.argv[1])
from oracle import hstu_oracle as O
from hstu_sequential_transduction_causal_b200 import hstu as H, workloads as W
from hstu_sequential_transduction_causal_b200.runtime import DeviceLayer, JaggedBatch, LayerRunner, to_dev, workspace
assert H.library_path().endswith("libhstu_debug.so"), H.library_path()
thr = O.time_bucket_thresholds(128)
wl = W.make_workload("c2", seed=5, lengths=[1, 127, 0, 129, 300, 513], D=256, H=4, N=600, pos_max_len=600,
                     backward=True)
jag = JaggedBatch(wl.offsets, wl.timestamps)
layer = DeviceLayer.upload(wl.layers[0], wl.D, wl.H, True)
run = LayerRunner(layer, jag, 1.0 / wl.N, wl.pos_max_len, torch.bfloat16, torch.bfloat16, keep_z=True)
x = to_dev(wl.x, torch.bfloat16)
y = run.forward(x).float().cpu().numpy()
D = wl.D
grads = [torch.zeros(n, dtype=torch.float32, device="cuda")
         for n in (4 * D * D, 4 * D, D * D, D, D, D, 2 * wl.pos_max_len - 1, 128)]
dx = torch.empty(wl.T, D, dtype=torch.bfloat16, device="cuda")
ws = workspace(H.hstu_layer_bwd_workspace_size(run.desc, jag.struct))
H.hstu_layer_bwd(run.desc, jag.struct, run.weights, x, None, run.saved_struct, to_dev(wl.dy, torch.bfloat16), None,
                 dx, None, H.layer_grads(*grads), ws)
torch.cuda.synchronize()
st = (run.device_status(), H.hstu_sync_status(ws))
assert st == (0, 0), st
ye, _ = O.layer_fwd(wl.x, wl.layers[0], wl.offsets, wl.timestamps, wl.H, 1.0 / wl.N, wl.pos_max_len, thr)
err = np.abs(y - ye) - (1e-2 + 1e-2 * np.abs(ye))
assert (err <= 0).all(), float(err.max())
# the richer bias: per-head tables and a token-type term (type gathers are checked too)
rng = np.random.default_rng(6)
Hh, d, L = 2, 64, 600
off, ts = wl.offsets, wl.timestamps
T = int(off[-1])
q, k, v = [(a / (1 + np.exp(-a))).astype(np.float16) for a in rng.standard_normal((3, T, Hh * d))]
rp = rng.standard_normal((Hh, 2 * L - 1)).astype(np.float32)
rt = rng.standard_normal((Hh, 128)).astype(np.float32)
types = rng.integers(0, 3, size=T).astype(np.int32)
ty = rng.standard_normal((Hh, 3, 3)).astype(np.float32)
desc = H.make_attn_desc(Hh, d, d, 1.0 / 512, L, H.HSTU_F16, Hh * d, Hh * d, Hh * d, Hh * d)
dty, dtt = to_dev(types, torch.int32), to_dev(ty, torch.float32)
ext = H.make_rab_ext(True, 3, dty, dtt)
ws2 = workspace(H.hstu_attn_ext_workspace_size(desc, jag.struct, ext))
out = torch.full((T, Hh * d), float("nan"), dtype=torch.float32, device="cuda")
H.hstu_attn_fwd_ext(desc, jag.struct, ext, *(to_dev(a, torch.float16) for a in (q, k, v)), to_dev(rp, torch.float32),
                    to_dev(rt, torch.float32), out, ws2)
torch.cuda.synchronize()
assert H.hstu_sync_status(ws2) == 0
exp = O.pointwise_attention_fwd_ext(*(a.astype(np.float64).reshape(T, Hh, d) for a in (q, k, v)), off, ts, rp, rt,
                                    1.0 / 512, L, thr, token_type=types, rab_type=ty, per_head=True).reshape(T, Hh * d)
scale = float(np.sqrt(np.mean(exp ** 2)))
err = np.abs(out.cpu().numpy() - exp) - (1e-2 * scale + 1e-2 * np.abs(exp))
assert (err <= 0).all(), float(err.max())
print("debug build ok")
"""


def test_checked_index_build_runs_clean_and_matches_the_oracle():
    from hstu_sequential_transduction_causal_b200 import build
    build.build(debug=True)
    env = dict(os.environ, HSTU_DEBUG="1")
    r = subprocess.run([sys.executable, "-c", _CHILD, ROOT], env=env, capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "debug build ok" in r.stdout


def test_values_beyond_the_fp16_range_are_reported():
    """BF16 mode keeps Z, SiLU(Z) and the attention weights in fp16: a pre-activation or a score past
    65504 is reported as HSTU_ERR_DEVICE; the same call inside the range reports nothing."""
    T, D = 64, 256
    for big, expect in ((300.0, H.HSTU_ERR_DEVICE), (100.0, 0)):
        x = np.zeros((T, D), np.float32)
        x[3, 0] = big
        W1 = np.zeros((4 * D, D), np.float32)
        W1[:, 0] = big                      # z[3, :] = big^2: 90000 or 10000
        uvqk = torch.empty(T, 4 * D, dtype=torch.float16, device="cuda")
        z = torch.empty(T, 4 * D, dtype=torch.float16, device="cuda")
        ws = workspace(256)
        H.hstu_uvqk_fwd(T, D, H.HSTU_BF16, H._dtype_code(uvqk), to_dev(x, torch.bfloat16), D,
                        to_dev(W1, torch.bfloat16), torch.zeros(4 * D, device="cuda"), uvqk, z, ws)
        assert H.hstu_sync_status(ws) == expect, big
    # scores q.k = 64 * 40^2 = 102400 (fp16 inputs in range, the score is not)
    for val, expect in ((40.0, H.HSTU_ERR_DEVICE), (4.0, 0)):
        off = W.offsets_from_lengths([130, 7])
        Tq, Hh, d, L = int(off[-1]), 1, 64, 256
        jag = JaggedBatch(off, np.arange(Tq, dtype=np.int64))
        desc = H.make_attn_desc(Hh, d, d, 1.0 / 256, L, H.HSTU_F16, d, d, d, d)
        qkv = torch.full((Tq, d), val, dtype=torch.float16, device="cuda")
        out = torch.empty(Tq, d, dtype=torch.float32, device="cuda")
        ws = workspace(H.hstu_attn_workspace_size(desc, jag.struct))
        H.hstu_attn_fwd(desc, jag.struct, qkv, qkv, qkv, torch.zeros(2 * L - 1, device="cuda"),
                        torch.zeros(128, device="cuda"), out, ws)
        assert H.hstu_sync_status(ws) == expect, val
