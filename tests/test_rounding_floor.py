"""Where the stated bf16 bound stops being reachable, shown on the CPU.

The bound for bf16 outputs is |d| <= 1e-2 + 1e-2 |ref|. The layer's weight gradients are sums over
thousands of tokens (rms ~34 for dW1 on the long-sequence workload), so an absolute term of 1e-2
is far below their rounding noise. These tests use ``tests/_rounding.py`` (the oracle with values
rounded to fp16 where the CUDA path stores them) to show that:
  - with no rounding the model is the oracle (so it is the oracle's arithmetic plus rounding);
  - rounding only q, k and v, the operands of the attention's tensor-core contractions, already
    puts thousands of dW1 and dW2 elements outside the bound on the long-sequence workload, while
    dX stays inside it: no implementation with 16-bit attention operands meets the bound for every
    weight-gradient element, and the GPU tests hold those elements to the model's count instead.
"""
import numpy as np

from oracle import hstu_oracle as O
from hstu_sequential_transduction_causal_b200 import workloads as W
from tests import _rounding as R

THR = O.time_bucket_thresholds(128)


def test_model_without_rounding_is_the_oracle():
    wl = W.make_workload("c4", seed=5, lengths=[40, 1, 0, 70], D=128, H=2, layers=2, N=128, pos_max_len=128)
    rng = np.random.default_rng(1)
    x = rng.standard_normal((wl.T, wl.D))
    dy = rng.standard_normal((wl.T, wl.D))
    ident = R.rounder(())
    y, dx, grads = R.stack_fwd_bwd(x, wl.layers, wl.offsets, wl.timestamps, wl.H, 1 / wl.N, wl.pos_max_len, dy,
                                   ident)
    xs, saved = [x], []
    for p in wl.layers:
        yl, sv = O.layer_fwd(xs[-1], p, wl.offsets, wl.timestamps, wl.H, 1 / wl.N, wl.pos_max_len, THR)
        xs.append(yl)
        saved.append(sv)
    g = dy
    ref = [None, None]
    for i in (1, 0):
        ref[i] = O.layer_bwd(g, wl.layers[i], saved[i], wl.offsets, wl.timestamps, wl.H, 1 / wl.N, wl.pos_max_len,
                             THR)
        g = ref[i]["dx"]
    assert np.allclose(y, xs[-1], rtol=1e-12, atol=1e-12)
    assert np.allclose(dx, g, rtol=1e-12, atol=1e-12)
    for i in (0, 1):
        for name in ("dW1", "db1", "dW2", "db2", "dgamma", "dbeta", "drab_pos", "drab_time"):
            assert np.allclose(grads[i][name], ref[i][name], rtol=1e-11, atol=1e-11), (i, name)


def test_rounding_only_the_attention_operands_breaks_the_bound_on_weight_gradients():
    wl = W.make_workload("c3", seed=0)
    args = (wl.offsets, wl.timestamps, wl.H, 1 / wl.N, wl.pos_max_len)
    p = wl.layers[0]
    _, sv = R.layer_fwd(wl.x, p, *args, R.rounder(()))
    exact = R.layer_bwd(wl.dy, p, sv, *args, R.rounder(()))
    # q, k, v are the column blocks 1..3 of U|V|Q|K: round those blocks only
    D = wl.D
    sv16 = dict(sv)
    s = sv["s"].copy()
    s[:, D:] = R.f16(s[:, D:])
    sv16["s"] = s
    T, d = wl.T, D // wl.H
    q, k, v = s[:, 2 * D:3 * D], s[:, 3 * D:], s[:, D:2 * D]
    sv16["o"] = O.pointwise_attention_fwd(q.reshape(T, wl.H, d), k.reshape(T, wl.H, d), v.reshape(T, wl.H, d),
                                          wl.offsets, wl.timestamps, p.rab_pos, p.rab_time, 1 / wl.N,
                                          wl.pos_max_len, THR).reshape(T, D)
    g, mu, rstd = O.norm_gate_fwd(sv16["o"], s[:, :D], p.gamma, p.beta)
    sv16.update(g=g, mu=mu, rstd=rstd)
    rounded = R.layer_bwd(wl.dy, p, sv16, *args, R.rounder(()))
    miss = {k: R.misses(rounded[k], exact[k]) for k in ("dx", "dW1", "dW2")}
    assert miss["dx"] == 0
    assert miss["dW1"] > 1000 and miss["dW2"] > 500, miss
