"""GPU parity of Stochastic Length (bit-exact integer work) and of the 8-layer stacked encoder on an
fp32 residual stream, forward and backward, against the oracle.

The oracle runs the same composition: Stochastic Length on the raw batch, then layer_fwd eight
times, then layer_bwd in reverse with each layer's dX as the previous layer's dY. Sequences are
independent, so the full-size workload is checked on sampled sequences run alone in the oracle.
"""
import numpy as np
import pytest
import torch

from oracle import hstu_oracle as O
from hstu_sequential_transduction_causal_b200 import hstu as H
from hstu_sequential_transduction_causal_b200 import workloads as W
from hstu_sequential_transduction_causal_b200.runtime import (DeviceLayer, Encoder, JaggedBatch, stochastic_length,
                                                              to_dev, workspace)
from tests import _rounding as R
from tests._util import BF16_TOL, THR, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from hstu_sequential_transduction_causal_b200 import build
    build.build()
    H.lib()
    torch.cuda.init()


def test_stochastic_length_bit_exact_with_ties():
    rng = np.random.default_rng(21)
    lengths = [0, 1, 2, 3, 7, 512, 600, 4096, 1000, 33]
    off = W.offsets_from_lengths(lengths)
    T = int(off[-1])
    ts = W.draw_timestamps(rng, lengths)
    keys = rng.integers(-20, 20, size=T).astype(np.int64)            # many ties, negative keys
    keys[int(off[8]):int(off[9])] = 5                                  # one sequence of equal keys
    x = rng.standard_normal((T, 64)).astype(np.float32)
    raw = JaggedBatch(off, ts)
    jag, kept, xk = stochastic_length(raw, to_dev(keys, torch.int64), 1.6, to_dev(x, torch.float32))
    new_off, kept_ref = O.stochastic_length(off, keys, 1.6)
    assert np.array_equal(jag.offsets_np, new_off)
    assert np.array_equal(kept.cpu().numpy(), kept_ref)
    assert np.array_equal(jag.timestamps.cpu().numpy(), ts[kept_ref])
    assert np.array_equal(xk.cpu().numpy(), x[kept_ref])


def test_stochastic_length_keep_count_every_length():
    lengths = np.arange(0, 8193, dtype=np.int64)
    off = torch.from_numpy(W.offsets_from_lengths(lengths)).cuda()
    raw = H.make_jagged(off, torch.zeros(1, dtype=torch.int64, device="cuda"), 8192)
    raw.T = int(lengths.sum())
    new_off = torch.empty(len(lengths) + 1, dtype=torch.int64, device="cuda")
    ws = workspace(256)
    H.hstu_stochastic_length_offsets(raw, 1.6, new_off, ws)
    got = np.diff(new_off.cpu().numpy())
    assert H.hstu_sync_status(ws) == 0
    exp = np.array([O.stochastic_length_keep(int(n), 1.6) for n in lengths])
    assert np.array_equal(got, exp)


def _oracle_encoder(x, layers, off, ts, H_, inv_N, L, dy):
    """Oracle composition: forward through the stack, backward in reverse. Returns
    (y, dx, [per-layer gradient dicts])."""
    acts = []
    for p in layers:
        y, sv = O.layer_fwd(x, p, off, ts, H_, inv_N, L, THR)
        acts.append(sv)
        x = y
    g = dy
    grads = [None] * len(layers)
    for l in reversed(range(len(layers))):
        r = O.layer_bwd(g, layers[l], acts[l], off, ts, H_, inv_N, L, THR)
        grads[l] = r
        g = r["dx"]
    return x, g, grads


NAMES = ("dW1", "db1", "dW2", "db2", "dgamma", "dbeta", "drab_pos", "drab_time")


def _run_encoder(wl, raw_x, raw_dy, sample=None):
    raw = JaggedBatch(wl.offsets, wl.timestamps)
    jag, kept, xk = stochastic_length(raw, to_dev(wl.extra["sl_keys"], torch.int64), wl.extra["sl_alpha"],
                                      to_dev(raw_x, torch.float32))
    layers = [DeviceLayer.upload(p, wl.D, wl.H, True) for p in wl.layers]
    enc = Encoder(layers, jag, 1.0 / wl.N, wl.pos_max_len)
    y = enc.forward(xk).clone()
    dy = to_dev(raw_dy, torch.float32)[kept]
    dx = enc.backward(dy).clone()
    torch.cuda.synchronize()
    assert enc.device_status() == 0
    return jag, kept.cpu().numpy(), y.cpu().numpy(), dx.cpu().numpy(), enc


def _rel(g, e):
    n = float(np.linalg.norm(e))
    return float(np.linalg.norm(np.asarray(g, np.float64) - e)) / n if n > 0 else 0.0


def _misses(g, e):
    return int((np.abs(np.asarray(g, np.float64) - e) > 1e-2 + 1e-2 * np.abs(e)).sum())


def _check_grads(got_views, ref, model, tag):
    """Every gradient: the count of elements outside the stated bound within R.miss_ceiling of the
    rounding model's count (tests/_rounding.py) and the norm-relative error within 1e-2; the weight
    gradients also element by element within the bound taken in units of their scale."""
    for name, g in zip(NAMES, got_views):
        e = np.asarray(ref[name], np.float64)
        g = (g.cpu().numpy() if hasattr(g, "cpu") else np.asarray(g)).reshape(e.shape)
        scale = max(1.0, float(np.sqrt(np.mean(e ** 2)))) if e.size else 1.0
        got_m, model_m = _misses(g, e), _misses(model[name], e)
        assert got_m <= R.miss_ceiling(model_m, e.size), (tag, name, got_m, model_m)
        if name not in ("drab_pos", "drab_time"):
            assert_close(g, e, 1e-2 * scale, 1e-2, what=f"{tag} {name}")
        assert _rel(g, e) <= 1e-2, (tag, name, _rel(g, e))


def test_encoder_eight_layers_fwd_bwd():
    """End to end through 8 layers, and every layer on the oracle's own input to that layer.

    Through a stack of LayerNorm layers with random weights a perturbation grows by about 1.35x per
    layer, so fp16 storage (tests/_rounding.py) alone takes some of the stack's outputs outside the
    elementwise bf16 bound. End to end, Y, dX and every layer's gradients are held to: the count of
    elements outside the bound within R.miss_ceiling of the rounding model's count on the same
    batch, and norm-relative error <= 1e-2. Each layer on the oracle's input to that layer (its
    forward input and its backward dY, computed by the oracle from the batch): Y element by element
    within the bound, dX and the gradients as above."""
    wl = W.make_workload("c4", seed=7, lengths=[700, 530, 5, 1])
    rng = np.random.default_rng(8)
    raw_x = rng.standard_normal((wl.T, wl.D)).astype(np.float32)
    raw_dy = rng.standard_normal((wl.T, wl.D)).astype(np.float32)
    jag, kept, y, dx, enc = _run_encoder(wl, raw_x, raw_dy)
    off, _ = O.stochastic_length(wl.offsets, wl.extra["sl_keys"], wl.extra["sl_alpha"])
    ts = wl.timestamps[kept]
    inv_N = 1.0 / wl.N
    # oracle, end to end, keeping every layer's input and upstream gradient
    xs, acts = [raw_x[kept].astype(np.float64)], []
    for p in wl.layers:
        yl, sv = O.layer_fwd(xs[-1], p, off, ts, wl.H, inv_N, wl.pos_max_len, THR)
        acts.append(sv)
        xs.append(yl)
    dys = [None] * len(wl.layers) + [raw_dy[kept].astype(np.float64)]
    grads_ref = [None] * len(wl.layers)
    for l in reversed(range(len(wl.layers))):
        grads_ref[l] = O.layer_bwd(dys[l + 1], wl.layers[l], acts[l], off, ts, wl.H, inv_N, wl.pos_max_len, THR)
        dys[l] = grads_ref[l]["dx"]
    ym, dxm, grads_m = R.stack_fwd_bwd(raw_x[kept], wl.layers, off, ts, wl.H, inv_N, wl.pos_max_len, raw_dy[kept])
    report = {"Y": (_misses(y, xs[-1]), _misses(ym, xs[-1])), "dX": (_misses(dx, dys[0]), _misses(dxm, dys[0]))}
    for key, size in (("Y", y.size), ("dX", dx.size)):
        assert report[key][0] <= R.miss_ceiling(report[key][1], size), (key, report[key])
    assert _rel(y, xs[-1]) <= 1e-2 and _rel(dx, dys[0]) <= 1e-2
    for l in range(len(wl.layers)):
        for name, g in zip(NAMES, enc.grads[l]):
            e = np.asarray(grads_ref[l][name], np.float64)
            gn = g.cpu().numpy().reshape(e.shape)
            assert _rel(gn, e) <= 1e-2, (l, name, _rel(gn, e))
            report[f"L{l} {name}"] = (_misses(gn, e), _misses(grads_m[l][name], e))
            assert report[f"L{l} {name}"][0] <= R.miss_ceiling(report[f"L{l} {name}"][1], e.size), \
                (l, name, report[f"L{l} {name}"])
    print("\nstack end to end, elements outside the stated bound (GPU, rounding model):",
          {k: v for k, v in report.items() if v != (0, 0)})
    # every layer on the oracle's own input
    layers = [DeviceLayer.upload(p, wl.D, wl.H, True) for p in wl.layers]
    one = Encoder([layers[0]], jag, inv_N, wl.pos_max_len)
    for l in range(len(wl.layers)):
        one.layers, one.weights = [layers[l]], [layers[l].weights()]
        x_l = xs[l].astype(np.float32)
        dy_l = dys[l + 1].astype(np.float32)
        yl_ref, sv = O.layer_fwd(x_l, wl.layers[l], off, ts, wl.H, inv_N, wl.pos_max_len, THR)
        gl_ref = O.layer_bwd(dy_l, wl.layers[l], sv, off, ts, wl.H, inv_N, wl.pos_max_len, THR)
        _, svm = R.layer_fwd(x_l, wl.layers[l], off, ts, wl.H, inv_N, wl.pos_max_len)
        gl_m = R.layer_bwd(dy_l, wl.layers[l], svm, off, ts, wl.H, inv_N, wl.pos_max_len)
        y_gpu = one.forward(to_dev(x_l, torch.float32)).clone()
        dx_gpu = one.backward(to_dev(dy_l, torch.float32)).clone()
        torch.cuda.synchronize()
        assert one.device_status() == 0
        assert_close(y_gpu.cpu().numpy(), yl_ref, *BF16_TOL, what=f"layer {l} Y")
        dxg = dx_gpu.cpu().numpy()
        assert _misses(dxg, gl_ref["dx"]) <= R.miss_ceiling(_misses(gl_m["dx"], gl_ref["dx"]), dxg.size), l
        dscale = max(1.0, float(np.sqrt(np.mean(gl_ref["dx"] ** 2))))
        assert_close(dxg, gl_ref["dx"], 1e-2 * dscale, 1e-2, what=f"layer {l} dX")
        _check_grads(one.grads[0], gl_ref, gl_m, f"layer {l}")


def test_encoder_stacked_workload_sampled_sequences():
    """64 raw sequences U[512, 4096] subsampled to n^0.8, 8 layers, d_model 512, all on the GPU.
    Three sequences run alone in the oracle: the first layer's output elementwise, the stack's
    output and dX by norm-relative error (see the test above)."""
    wl = W.make_workload("c4", seed=0)
    rng = np.random.default_rng(9)
    raw_x = W.round_bf16(rng.standard_normal((wl.T, wl.D)))
    raw_dy = rng.standard_normal((wl.T, wl.D)).astype(np.float32)
    jag, kept, y, dx, enc = _run_encoder(wl, raw_x, raw_dy)
    y0 = enc.xs[1].cpu().numpy()
    new_off = jag.offsets_np
    for b in (0, 17, 63):
        s, e = int(new_off[b]), int(new_off[b + 1])
        rows = kept[s:e]
        off_b = np.array([0, e - s], np.int64)
        y0_ref, _ = O.layer_fwd(raw_x[rows], wl.layers[0], off_b, wl.timestamps[rows], wl.H, 1.0 / wl.N,
                                wl.pos_max_len, THR)
        assert_close(y0[s:e], y0_ref, *BF16_TOL, what=f"first layer Y, sequence {b}")
        y_ref, dx_ref, _ = _oracle_encoder(raw_x[rows], wl.layers, off_b, wl.timestamps[rows], wl.H, 1.0 / wl.N,
                                           wl.pos_max_len, raw_dy[rows])
        ym, dxm, _ = R.stack_fwd_bwd(raw_x[rows], wl.layers, off_b, wl.timestamps[rows], wl.H, 1.0 / wl.N,
                                     wl.pos_max_len, raw_dy[rows])
        assert _rel(y[s:e], y_ref) <= 1e-2, (b, _rel(y[s:e], y_ref))
        assert _rel(dx[s:e], dx_ref) <= 1e-2, (b, _rel(dx[s:e], dx_ref))
        miss = {"Y": (_misses(y[s:e], y_ref), _misses(ym, y_ref)), "dX": (_misses(dx[s:e], dx_ref), _misses(dxm, dx_ref))}
        for key, (g_m, m_m) in miss.items():
            assert g_m <= R.miss_ceiling(m_m, y_ref.size), (b, key, g_m, m_m)
        print(f"\nsequence {b}: elements outside the stated bound (GPU, rounding model): {miss}")
