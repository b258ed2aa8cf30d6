"""Throughput of the HSTU layer hot path on B200; one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c3|c2] [--impl ours|reference]

Default workload: one HSTU layer forward + backward (bf16) over 8 jagged sequences with Pareto(1.2)
lengths clipped to [256, 8192], d_model 512, 8 heads (seed = rank). A step is the whole layer:
f1 + SiLU (U|V|Q|K), jagged causal pointwise attention, LayerNorm (.) U, f2 + residual, then the
full backward (weight, bias and table gradients, dX). Inputs are resident in HBM; the L2 is flushed
(a 512 MB write) before every timed step; each step is bracketed by CUDA events on the launching
stream and the summed device time is taken as the max over ranks. Under torchrun each rank takes
its own batch (weak scaling) and the step ends with an NCCL all-reduce of the gradients, the one
exchange a data-parallel training step has.

``--impl reference`` times the CPU oracle (plain numpy fp64) on a bounded sample of the same
workload on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "HSTU layer jagged tokens/sec (bf16 fwd/bwd); attention TFLOP/s as % of bf16 peak"
WORKLOADS = {
    "c3": dict(backward=True, B=8,
               desc="HSTU layer forward+backward bf16: B=8 jagged sequences per GPU, lengths Pareto(alpha=1.2) "
                    "clipped to [256,8192], d_model 512, H 8, d_qk=d_v=64, N=8192, rab_pos for max_len 8192; one "
                    "global batch of 8 x n_gpus sequences (seed 0) split over the GPUs by hstu_dp_partition"),
    "c2": dict(backward=False, B=32,
               desc="HSTU layer forward bf16: B=32 jagged sequences per GPU, lengths U[64,1024], d_model 256, H 4, "
                    "d_qk=d_v=64, N=1024; one global batch of 32 x n_gpus sequences (seed 0) split over the GPUs "
                    "by hstu_dp_partition"),
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """Samples nvidia-smi SM clocks and throttle reasons every 100 ms (timestamped)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.proc = None
        self.window = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.samples.append((time.time(), parts))

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sel = self.samples
        if self.window:
            inside = [s for s in self.samples if self.window[0] <= s[0] <= self.window[1]]
            sel = inside or self.samples
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(s[1][1]) for s in sel if num(s[1][1]) is not None]
        mx = [num(s[1][2]) for s in sel if num(s[1][2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, s in sel for i in range(4) if s[5 + i].lower() == "active"})
        inside = bool(self.window) and any(self.window[0] <= s[0] <= self.window[1] for s in self.samples)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(sel),
                "window": "timed region" if inside else "warm-up + timed"}


def attn_flops(offsets: np.ndarray, D: int) -> float:
    """Algorithmic attention forward flops: 2 D sum_b n_b (n_b + 1) (causal pairs only, QK^T and PV)."""
    n = np.diff(offsets).astype(np.float64)
    return float(2.0 * D * np.sum(n * (n + 1)))


def kernel_source_sha(path: str, signature: str) -> str:
    """sha256 (16 hex digits) of one kernel's source text: from its signature to the first closing
    brace at column 0 after it."""
    text = open(path).read()
    i = text.index(signature)
    j = text.index("\n}\n", i)
    return hashlib.sha256(text[i:j + 3].encode()).hexdigest()[:16]


def traffic_record(name: str):
    """ncu DRAM bytes per attention launch from profiles/, valid only while the persistent kernel's
    source is the one the counters were taken on."""
    p = os.path.join(ROOT, "profiles", f"attn_fwd_{name}.traffic.json")
    src = os.path.join(ROOT, "hstu_sequential_transduction_causal_b200", "csrc", "attn_fwd2_sm100.cu")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    sha = kernel_source_sha(src, "attn_fwd_persistent_kernel(const __grid_constant__")
    return rec.get("dram_bytes_per_launch") if rec.get("kernel_sha") == sha else None


def cpu_oracle_sample(wl, backward: bool, budget_s: float = 12.0):
    """Times the oracle layer (forward, and backward when the workload has one) sequence by
    sequence, cycling through the batch, until about budget_s seconds (at least one sequence);
    returns tokens/s on the host's cores."""
    from oracle import hstu_oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:  # noqa: BLE001
        cores = 1
    thr = O.time_bucket_thresholds(128)
    p = wl.layers[0]
    tokens = seqs = 0
    t0 = time.perf_counter()
    while True:
        b = seqs % wl.B
        s, e = int(wl.offsets[b]), int(wl.offsets[b + 1])
        off = np.array([0, e - s], np.int64)
        y, sv = O.layer_fwd(wl.x[s:e], p, off, wl.timestamps[s:e], wl.H, 1.0 / wl.N, wl.pos_max_len, thr)
        if backward:
            O.layer_bwd(wl.dy[s:e], p, sv, off, wl.timestamps[s:e], wl.H, 1.0 / wl.N, wl.pos_max_len, thr)
        tokens += e - s
        seqs += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    what = "layer forward+backward" if backward else "layer forward"
    return {"value": tokens / dt, "unit": "tokens/s", "cores": int(cores), "kind": "oracle",
            "sample": f"{seqs} sequences cycling through the {wl.B} of the batch ({tokens} tokens), numpy fp64 "
                      f"{what}, {dt:.1f} s wall"}


def run_reference(args, rank, world):
    from hstu_sequential_transduction_causal_b200 import workloads as W
    if rank != 0:
        return
    wl = W.make_workload(args.workload, seed=0)
    bwd = WORKLOADS[args.workload]["backward"]
    vals = []
    r = None
    # the whole reference run stays within about two minutes of oracle time
    per_step = min(args.ref_budget, 120.0 / max(1, args.warmup + args.steps))
    for i in range(args.warmup + args.steps):
        r = cpu_oracle_sample(wl, bwd, budget_s=per_step)
        if i >= args.warmup:
            vals.append(r["value"])
    value = float(np.median(vals))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOADS[args.workload]["desc"], "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
                             "sample": r["sample"]},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def grad_buffer(D: int, pos_max_len: int, device):
    """One flat fp32 buffer holding a layer's eight gradients (dW1, db1, dW2, db2, dgamma, dbeta,
    drab_pos, drab_time), each view on a 16-byte boundary; a data-parallel step all-reduces it once."""
    import torch
    sizes = [4 * D * D, 4 * D, D * D, D, D, D, 2 * pos_max_len - 1, 128]
    padded = [(n_ + 3) // 4 * 4 for n_ in sizes]
    flat = torch.zeros(sum(padded), dtype=torch.float32, device=device)
    views, o = [], 0
    for n_, pn in zip(sizes, padded):
        views.append(flat[o:o + n_])
        o += pn
    return flat, views


def reduce_over_ranks(total_ms: float, attn_ms: float, tokens: int, world: int, device):
    """Max over ranks of the device times, sum over ranks of the tokens (weak scaling: each rank
    processes its own batch)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([total_ms, attn_ms], dtype=torch.float64, device=device)
    n = torch.tensor([float(tokens)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(n)
    return float(t[0]), float(t[1]), float(n.item())


def measure_other_workloads(dev):
    """Throughput of the two other workloads the hot path serves, on this GPU (CUDA events):
    the 8-layer encoder forward+backward with Stochastic Length (64 raw sequences U[512, 4096],
    alpha 1.6, d_model 512, H 8; tokens/s after subsampling) and M-FALCON ranking (16 users x
    2048-token prefixes, 1024 candidates each in micro-batches of 256, 4 layers; candidates/s with
    the prefix K/V built in the call, and with it reused from the cache)."""
    import torch
    from hstu_sequential_transduction_causal_b200 import hstu as H
    from hstu_sequential_transduction_causal_b200 import workloads as W
    from hstu_sequential_transduction_causal_b200.runtime import (DeviceLayer, Encoder, JaggedBatch, stochastic_length,
                                                                  to_dev, workspace)
    out = {}
    stream = torch.cuda.current_stream()

    def timed(fn, warm=2, reps=5):
        for _ in range(warm):
            fn()
        torch.cuda.synchronize()
        ms = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            ms.append(e0.elapsed_time(e1))
        return float(np.median(ms))

    wl = W.make_workload("c4", seed=0)
    rng = np.random.default_rng(9)
    raw = JaggedBatch(wl.offsets, wl.timestamps, device=dev)
    raw_x = to_dev(rng.standard_normal((wl.T, wl.D)).astype(np.float32), torch.float32, dev)
    jag, kept, xk = stochastic_length(raw, to_dev(wl.extra["sl_keys"], torch.int64, dev), wl.extra["sl_alpha"],
                                      raw_x, device=dev)
    layers = [DeviceLayer.upload(p, wl.D, wl.H, True, device=dev) for p in wl.layers]
    enc = Encoder(layers, jag, 1.0 / wl.N, wl.pos_max_len, device=dev)
    dy = torch.randn(jag.T, wl.D, dtype=torch.float32, device=dev)

    def enc_step():
        enc.forward(xk)
        enc.backward(dy)
    ms = timed(enc_step)
    if enc.device_status() != 0:
        raise RuntimeError("device status error in the encoder leg")
    out["encoder_8_layers_fwd_bwd"] = {"value": jag.T / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
                                       "tokens": jag.T, "raw_tokens": wl.T,
                                       "workload": "64 sequences U[512,4096] -> Stochastic Length alpha 1.6, "
                                                   "8 layers, d_model 512, H 8, fp32 residual stream, eager launches"}
    del enc, layers, raw_x, xk, dy
    fw = W.make_falcon_workload(seed=0)
    lens = np.diff(fw.prefix_offsets)
    pj = JaggedBatch(fw.prefix_offsets, fw.prefix_ts, max_len=int(lens.max()), device=dev)
    fl = [DeviceLayer.upload(p, fw.D, fw.H, True, device=dev) for p in fw.layers]
    fws = [x.weights() for x in fl]
    desc = H.make_falcon_desc(len(fl), fw.users, fw.m, fw.b_m, fw.D, fw.H, 1.0 / fw.N, fw.pos_max_len)
    px, cx = to_dev(fw.prefix_x, torch.bfloat16, dev), to_dev(fw.cand_x, torch.bfloat16, dev)
    req = to_dev(fw.request_ts, torch.int64, dev)
    cache = torch.empty(H.hstu_falcon_cache_size(desc, pj.struct) // 2, dtype=torch.float16, device=dev)
    fws_ws = workspace(H.hstu_falcon_workspace_size(desc, pj.struct), dev)
    fout = torch.empty(fw.users * fw.m, fw.D, dtype=torch.float32, device=dev)

    def falcon(valid):
        return lambda: H.hstu_falcon_fwd(desc, fws, pj.struct, px, cache, valid, None, cx, req, fout, fws_ws)
    ms_build = timed(falcon(0), reps=3)
    ms_reuse = timed(falcon(1), reps=3)
    if H.hstu_sync_status(fws_ws) != 0:
        raise RuntimeError("device status error in the M-FALCON leg")
    n_c = fw.users * fw.m
    out["falcon_ranking"] = {"value": n_c / (ms_build / 1e3), "unit": "candidates/s", "ms_per_request_batch": ms_build,
                             "cached_prefix": {"value": n_c / (ms_reuse / 1e3), "unit": "candidates/s",
                                               "ms": ms_reuse},
                             "workload": "16 users x 2048-token prefixes, 1024 candidates per user, micro-batches "
                                         "of 256, 4 layers, d_model 512, H 8"}
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="c3", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-budget", type=float, default=15.0)
    ap.add_argument("--no-extra", action="store_true", help="skip the encoder and M-FALCON throughput legs")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist

    from hstu_sequential_transduction_causal_b200 import hstu as H
    from hstu_sequential_transduction_causal_b200 import workloads as W
    from hstu_sequential_transduction_causal_b200.build import build
    from hstu_sequential_transduction_causal_b200.runtime import (DeviceLayer, JaggedBatch, LayerRunner, SavedActs,
                                                                  to_dev, workspace)

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    if rank == 0:
        build()
    if world > 1:
        dist.barrier()
    H.lib()
    stream = torch.cuda.current_stream()
    backward = WORKLOADS[args.workload]["backward"]

    # one global batch, split over the ranks by whole sequences (cost-balanced, the same split on
    # every rank); per-rank work stays about constant as the number of GPUs grows
    from hstu_sequential_transduction_causal_b200.runtime import shard_rows
    gwl = W.make_workload(args.workload, seed=0, B=WORKLOADS[args.workload]["B"] * world)
    if gwl.dy is None:
        gwl.dy = W.round_bf16(np.random.default_rng(1000).standard_normal((gwl.T, gwl.D)))
    rank_of, rank_cost = H.hstu_dp_partition(np.diff(gwl.offsets), gwl.D, world)
    shard_off, shard = shard_rows(gwl.offsets, rank_of, rank)
    wl = W.Workload(name=gwl.name, D=gwl.D, H=gwl.H, dtype=gwl.dtype, N=gwl.N, pos_max_len=gwl.pos_max_len,
                    offsets=shard_off, timestamps=gwl.timestamps[shard], x=gwl.x[shard], layers=gwl.layers,
                    dy=gwl.dy[shard])
    D, Hh, T = wl.D, wl.H, wl.T
    jag = JaggedBatch(wl.offsets, wl.timestamps, device=dev)
    layer = DeviceLayer.upload(wl.layers[0], D, Hh, True, device=dev)
    x = to_dev(wl.x, torch.bfloat16, dev)
    dy = to_dev(wl.dy, torch.bfloat16, dev)
    y = torch.empty(T, D, dtype=torch.bfloat16, device=dev)
    dx = torch.empty(T, D, dtype=torch.bfloat16, device=dev)
    adesc = H.make_attn_desc(Hh, D // Hh, D // Hh, 1.0 / wl.N, wl.pos_max_len, H.HSTU_F16, 4 * D, 4 * D, 4 * D, D)
    ldesc = H.make_layer_desc(D, Hh, 1.0 / wl.N, wl.pos_max_len, H.HSTU_BF16, H.HSTU_BF16, H.HSTU_BF16)
    # with a backward, the forward also writes the attention backward's bias tiles (saved.attn_bias)
    sv = SavedActs.empty(T, D, torch.bfloat16, keep_z=backward, device=dev,
                         bias_cache_bytes=H.hstu_layer_bias_cache_size(ldesc, jag.struct) if backward else 0)
    svs = sv.struct()
    ws = workspace(max(H.hstu_attn_workspace_size(adesc, jag.struct), H.hstu_layer_workspace_size(ldesc, jag.struct),
                       H.hstu_layer_bwd_workspace_size(ldesc, jag.struct) if backward else 0), dev)
    flat, views = grad_buffer(D, wl.pos_max_len, dev)
    grads = H.layer_grads(*views)
    weights = layer.weights()
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.zeros(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        """Evicts the step's data from the 126 MB L2: a 512 MB write, then a 256 MB read so that the
        lines left behind are clean (the step does not pay the flush's own write-backs)."""
        flush.zero_()
        torch.sum(flush_rd, dim=0, out=flush_sink)
    # kernels of ours per step (cross-checked against the ncu launch list in profiles/)
    # f1 GEMM (its launch also computes the attention's work list) | bias tiles (with the fp16 W2 copy
    # f2 reads), attention | LN-gate | f2 GEMM
    n_fwd_kernels = 5
    # fp16 dy with the db2 partial sums, the fp16 copies of x, W1, W2 and the zeroed accumulators (one
    # launch) | dG with dW2 (one grouped GEMM launch) | LN-gate bwd | attention bwd, table gradients (the
    # transposed bias tiles and the work list come from the forward's cache) | dZ with db1, and the
    # finish of db2, dgamma and dbeta (one launch) | dX with dW1 (one grouped launch)
    n_bwd_kernels = 7
    names = ["uvqk", "attn", "norm_gate", "out_proj"] + (["backward"] if backward else [])

    def attention_forward():
        H.hstu_attn_fwd(adesc, jag.struct, sv.uvqk[:, 2 * D:], sv.uvqk[:, 3 * D:], sv.uvqk[:, D:], layer.rab_pos,
                        layer.rab_time, sv.o, ws)

    # CUDA events the library records right around its dominant kernels (hstu_profile_events); captured
    # into the step graph as event nodes, read after every timed replay
    prof_kernels = [H.PROFILE_ATTN_FWD, H.PROFILE_NORM_FWD, H.PROFILE_BIAS] + (
        [H.PROFILE_ATTN_BWD, H.PROFILE_NORM_BWD, H.PROFILE_TABLE_GRAD, H.PROFILE_DZ] if backward else [])
    prof_ev = {k: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for k in prof_kernels}
    prof_ms = {k: [] for k in prof_kernels}

    # data parallelism: the gradient sum runs on a side stream, started by the events hstu_layer_bwd
    # records when dW2, db2, dgamma, dbeta, db1 and the tables are final (reduced while the launch that
    # computes dX and dW1 runs) and when dW1 is final
    comm = torch.cuda.Stream(device=dev) if world > 1 else None
    n_late = 4 * D * D + 4 * D             # dW1, db1 lead the flat buffer
    if comm is not None and backward:
        ev_early, ev_w1 = torch.cuda.Event(), torch.cuda.Event()
        H.hstu_layer_bwd_ready_events(ev_early, ev_w1)

    def reduce_grads(buf=None):
        buf = flat if buf is None else buf
        with torch.cuda.stream(comm):
            comm.wait_event(ev_early)
            dist.all_reduce(buf[n_late:])
            comm.wait_event(ev_w1)
            dist.all_reduce(buf[:n_late])
        stream.wait_stream(comm)

    # The timed step is one hstu_layer_fwd + hstu_layer_bwd (the forward also writes the backward's bias
    # tiles into the saved struct's cache). The per-piece breakdown runs the forward as its four entry
    # points instead, which write no cache: its backward gets a saved struct without one (and computes
    # its own bias tiles).
    svs_pieces = H.layer_saved(sv.uvqk, sv.z, sv.o, sv.g, sv.mu, sv.rstd)

    def step(ev=None, all_reduce=True):
        if ev is None:
            H.hstu_layer_fwd(ldesc, jag.struct, weights, x, None, y, None, svs, ws)
            if backward:
                H.hstu_layer_bwd(ldesc, jag.struct, weights, x, None, svs, dy, None, dx, None, grads, ws)
                if world > 1 and all_reduce:
                    reduce_grads()
            return
        rec = lambda i: ev[i].record(stream)
        rec(0)
        H.hstu_uvqk_fwd(T, D, H.HSTU_BF16, H.HSTU_F16, x, D, layer.W1, layer.b1, sv.uvqk, sv.z, ws)
        rec(1)
        attention_forward()
        rec(2)
        H.hstu_norm_gate_fwd(T, D, H.HSTU_F32, H.HSTU_F16, H.HSTU_F16, sv.o, D, sv.uvqk, 4 * D, layer.gamma,
                             layer.beta, 1e-5, sv.g, sv.mu, sv.rstd)
        rec(3)
        H.hstu_out_proj_fwd(T, D, H.HSTU_BF16, H.HSTU_F16, sv.g, layer.W2, layer.b2, x, H.HSTU_BF16, y, H.HSTU_BF16,
                            None, ws)
        rec(4)
        if backward:
            H.hstu_layer_bwd(ldesc, jag.struct, weights, x, None, svs_pieces, dy, None, dx, None, grads, ws)
            if world > 1 and all_reduce:
                reduce_grads()
            rec(5)

    clk = ClockSampler(local_rank)
    clk.__enter__()
    try:
        for _ in range(args.warmup):
            flush_l2()
            step()
        torch.cuda.synchronize()
        if H.hstu_sync_status(ws) != 0:
            raise RuntimeError("device status error during warm-up")
        # per-piece device times of eagerly launched steps (the breakdown in the JSON line)
        nev = len(names) + 1
        n_eager = min(args.steps, 20)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(n_eager)]
        for i in range(n_eager):
            flush_l2()
            step(evs[i])
        torch.cuda.synchronize()
        seg = np.array([[e[k].elapsed_time(e[k + 1]) for k in range(nev - 1)] for e in evs])   # ms
        # the timed steps replay one CUDA graph of the whole step (no host launch cost inside); the
        # gradient all-reduce of a multi-GPU run follows each replay on the same stream
        # one GPU: the timed steps replay one CUDA graph of the whole step (no host launch cost
        # inside); several GPUs: eager steps, so that the gradient all-reduce on the side stream
        # overlaps the end of the backward
        graph = torch.cuda.CUDAGraph() if world == 1 else None
        if graph is not None:
            with torch.cuda.graph(graph):
                step(all_reduce=False)
        attn_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(attn_graph):
            attention_forward()
        # the same step with the library's kernel events recorded around its dominant kernels (event
        # nodes cost some time between kernels, so the headline replays the graph without them)
        for k, (e0_, e1_) in prof_ev.items():
            H.hstu_profile_events(k, e0_, e1_)
        prof_graph = torch.cuda.CUDAGraph() if world == 1 else None
        if prof_graph is not None:
            with torch.cuda.graph(prof_graph):
                step(all_reduce=False)
            for k in prof_ev:
                H.hstu_profile_events(k)
        run_prof = prof_graph.replay if prof_graph is not None else step
        run_step = graph.replay if graph is not None else step
        for _ in range(3):
            flush_l2()
            run_step()
            attn_graph.replay()
        torch.cuda.synchronize()
        e_step = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t_start = time.time()
        if world > 1:
            for k in prof_ev:
                H.hstu_profile_events(k)
        for i in range(args.steps):
            flush_l2()
            e_step[i][0].record(stream)
            run_step()
            e_step[i][1].record(stream)
        torch.cuda.synchronize()
        t_end = time.time()
        clk.window = (t_start, t_end)
        # per-kernel device times: as many steps again, each followed by a read of the kernel events
        # (the next replay records them anew)
        if world > 1:
            for k, (e0_, e1_) in prof_ev.items():
                H.hstu_profile_events(k, e0_, e1_)
        for i in range(args.steps):
            flush_l2()
            run_prof()
            torch.cuda.synchronize()
            for k, (e0_, e1_) in prof_ev.items():
                prof_ms[k].append(e0_.elapsed_time(e1_))
        for k in prof_ev:
            H.hstu_profile_events(k)
        n_attn = 20
        e_attn = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_attn)]
        for i in range(n_attn):
            flush_l2()
            e_attn[i][0].record(stream)
            attn_graph.replay()
            e_attn[i][1].record(stream)
        torch.cuda.synchronize()
    finally:
        clk.__exit__()
    if world > 1:
        dist.barrier()
    st = H.hstu_sync_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st} in the timed region")
    total_ms = float(sum(a.elapsed_time(b) for a, b in e_step))
    attn_ms = float(np.mean([a.elapsed_time(b) for a, b in e_attn]))
    total_ms, attn_ms_max, tokens_all = reduce_over_ranks(total_ms, attn_ms, T, world, dev)
    value = tokens_all * args.steps / (total_ms / 1e3)

    # End to end through the public layer API: per step the host->device copy of the step's inputs
    # (x, dy, offsets, timestamps) from pinned memory, hstu_layer_fwd (+ hstu_layer_bwd), and the
    # device->host copy of the step's results (Y, and dX and the gradients). Pipelined as an input
    # pipeline runs: two buffer sets; step i's inputs are copied in on one stream while step i - 1
    # computes, and step i - 1's results are copied out on another while step i computes. The K
    # timed steps are one region (every step's copies inside it), timed on the compute stream.
    h_x = torch.from_numpy(wl.x).to(torch.bfloat16).pin_memory()
    h_dy = torch.from_numpy(wl.dy).to(torch.bfloat16).pin_memory()
    h_off = torch.from_numpy(wl.offsets).pin_memory()
    h_ts = torch.from_numpy(wl.timestamps).pin_memory()
    h_y = torch.empty(T, D, dtype=torch.bfloat16).pin_memory()
    h_dx = torch.empty(T, D, dtype=torch.bfloat16).pin_memory()
    h_grads = torch.empty_like(flat, device="cpu").pin_memory()
    bufs = []
    for _ in range(2):
        jb = JaggedBatch(wl.offsets, wl.timestamps, device=dev)
        rb = LayerRunner(layer, jb, 1.0 / wl.N, wl.pos_max_len, torch.bfloat16, torch.bfloat16, keep_z=backward,
                         device=dev)
        fb, vb = grad_buffer(D, wl.pos_max_len, dev)
        bufs.append(dict(jag=jb, run=rb, x=torch.empty(T, D, dtype=torch.bfloat16, device=dev),
                         dy=torch.empty(T, D, dtype=torch.bfloat16, device=dev),
                         dx=torch.empty(T, D, dtype=torch.bfloat16, device=dev), flat=fb, grads=H.layer_grads(*vb),
                         ws=workspace(H.hstu_layer_bwd_workspace_size(rb.desc, jb.struct) if backward else 256, dev),
                         ev_in=torch.cuda.Event(), ev_comp=torch.cuda.Event(), ev_out=torch.cuda.Event()))
    h2d_stream = torch.cuda.Stream(device=dev)
    d2h_stream = torch.cuda.Stream(device=dev)

    def e2e_step(i):
        b = bufs[i % 2]
        with torch.cuda.stream(h2d_stream):
            if i >= 2:
                h2d_stream.wait_event(b["ev_comp"])   # step i - 2 has consumed this set's inputs
            b["jag"].offsets.copy_(h_off, non_blocking=True)
            b["jag"].timestamps.copy_(h_ts, non_blocking=True)
            b["x"].copy_(h_x, non_blocking=True)
            b["dy"].copy_(h_dy, non_blocking=True)
            b["ev_in"].record(h2d_stream)
        stream.wait_event(b["ev_in"])
        if i >= 2:
            stream.wait_event(b["ev_out"])            # step i - 2's results have left this set
        r = b["run"]
        r.forward(b["x"])
        if backward:
            H.hstu_layer_bwd(r.desc, b["jag"].struct, r.weights, b["x"], None, r.saved_struct, b["dy"], None,
                             b["dx"], None, b["grads"], b["ws"])
            if world > 1:
                reduce_grads(b["flat"])
        b["ev_comp"].record(stream)
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(b["ev_comp"])
            h_y.copy_(r.y, non_blocking=True)
            if backward:
                h_dx.copy_(b["dx"], non_blocking=True)
                h_grads.copy_(b["flat"], non_blocking=True)
            b["ev_out"].record(d2h_stream)

    def e2e_run(k):
        for i in range(k):
            e2e_step(i)
        stream.wait_event(bufs[(k - 1) % 2]["ev_out"])
        stream.wait_event(bufs[k % 2]["ev_out"])

    e2e_run(4)
    torch.cuda.synchronize()
    n_e2e = max(10, args.steps // 4)
    flush_l2()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    e2e_run(n_e2e)
    e1.record(stream)
    e1.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    te = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(te, op=dist.ReduceOp.MAX)
    e2e_value = tokens_all * n_e2e / (float(te.item()) / 1e3)
    for b in bufs:
        if b["run"].device_status() != 0 or H.hstu_sync_status(b["ws"]) != 0:
            raise RuntimeError("device status error in the end-to-end pass")

    def same_size_copy_gbs(nbytes):
        """A torch device copy moving the same bytes (half read from cold memory, half written), timed
        with events like the kernels: the bandwidth a standalone kernel of this size reaches here."""
        n = int(nbytes) // 4 // 2 // 256 * 256
        src = torch.empty(n * 8, dtype=torch.float32, device=dev)   # eight regions: each copy reads cold data
        dst = torch.empty(n, dtype=torch.float32, device=dev)
        ts = []
        for i in range(12):
            flush_l2()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            dst.copy_(src[(i % 8) * n:(i % 8 + 1) * n])
            a1.record(stream)
            a1.synchronize()
            if i >= 2:
                ts.append(a0.elapsed_time(a1))
        del src, dst
        return 8.0 * n / (float(np.mean(ts)) / 1e3) / 1e9

    kern_ms = {k: float(np.mean(v)) for k, v in prof_ms.items()}
    if world > 1:
        tk = torch.tensor([kern_ms[k] for k in prof_kernels], dtype=torch.float64, device=dev)
        dist.all_reduce(tk, op=dist.ReduceOp.MAX)
        kern_ms = {k: float(tk[i]) for i, k in enumerate(prof_kernels)}
    extra = measure_other_workloads(dev) if (world == 1 and not args.no_extra) else None

    if rank == 0:
        peaks, peak_kind = load_peaks()
        flops = attn_flops(wl.offsets, D)
        tf_peak = float(peaks.get("bf16_tflops"))
        hbm_peak = float(peaks.get("hbm_gbs"))
        achieved = flops / (kern_ms[H.PROFILE_ATTN_FWD] / 1e3) / 1e12
        whole_fwd = flops / (attn_ms_max / 1e3) / 1e12
        # LayerNorm (.) U: O fp32 and U fp16 read, G fp16 written, mu and rstd fp32 written
        ln_bytes = T * (4 * D + 2 * D + 2 * D + 8)
        rooflines = {
            "attention_forward_whole": {
                "what": "work list + bias tiles + attention kernel (its own graph, L2 flushed before each replay)",
                "achieved": whole_fwd, "peak": tf_peak, "unit": "TFLOP/s", "frac": whole_fwd / tf_peak,
                "ms": attn_ms_max},
            "norm_gate_fwd": {"bound": "hbm", "achieved": ln_bytes / (kern_ms[H.PROFILE_NORM_FWD] / 1e3) / 1e9,
                              "peak": hbm_peak, "unit": "GB/s", "algorithmic_bytes_per_launch": ln_bytes,
                              "ms": kern_ms[H.PROFILE_NORM_FWD]}}
        rooflines["norm_gate_fwd"]["frac"] = rooflines["norm_gate_fwd"]["achieved"] / hbm_peak
        # kernels this short pay a fixed ramp and drain (about 5 us here) that the peak copy of a large
        # buffer does not: a device copy of the same bytes, timed the same way, is the reference they
        # can reach as a separate launch
        cpy = same_size_copy_gbs(ln_bytes)
        rooflines["norm_gate_fwd"]["same_size_copy"] = {
            "achieved": cpy, "unit": "GB/s", "frac": rooflines["norm_gate_fwd"]["achieved"] / cpy,
            "what": "torch device copy of the same bytes from cold memory, CUDA events"}

        def hbm_line(kernel, nbytes, what):
            a_ = nbytes / (kern_ms[kernel] / 1e3) / 1e9
            c_ = same_size_copy_gbs(nbytes)
            return {"bound": "hbm", "achieved": a_, "peak": hbm_peak, "unit": "GB/s", "frac": a_ / hbm_peak,
                    "algorithmic_bytes_per_launch": int(nbytes), "ms": kern_ms[kernel], "what": what,
                    "same_size_copy": {"achieved": c_, "unit": "GB/s", "frac": a_ / c_,
                                       "what": "torch device copy of the same bytes from cold memory, CUDA events"}}
        # causal 128 x 128 tile pairs (this workload packs no sequence)
        nt_b = (np.diff(wl.offsets) + 127) // 128
        n_pairs = int(np.sum(nt_b * (nt_b + 1) // 2))
        # bias tiles with the layer's cache: per pair the fp16 half-bias tile, its key-major copy and the
        # u8 buckets written; the fp16 W2 copy (read bf16, write fp16); the timestamps read
        rooflines["bias_tiles"] = hbm_line(H.PROFILE_BIAS, n_pairs * (32768 + 32768 + 16384) + 4 * D * D + 8 * T,
                                           f"{n_pairs} causal tile pairs: 80 KB written per pair, + W2 copy")
        if backward:
            # attention backward: four contractions (P recompute not counted) = 2x the forward's flops
            bw = 2 * flops / (kern_ms[H.PROFILE_ATTN_BWD] / 1e3) / 1e12
            rooflines["attention_backward"] = {"bound": "tensor", "achieved": bw, "peak": tf_peak, "unit": "TFLOP/s",
                                               "frac": bw / tf_peak, "algorithmic_flops_per_launch": 2 * flops,
                                               "ms": kern_ms[H.PROFILE_ATTN_BWD]}
            # its backward: dG fp32, O fp32, U and Z_U fp16, mu and rstd read; dO and dZ_U fp16 written
            lnb_bytes = T * (4 * D + 4 * D + 2 * D + 2 * D + 8 + 2 * D + 2 * D)
            a_ = lnb_bytes / (kern_ms[H.PROFILE_NORM_BWD] / 1e3) / 1e9
            rooflines["norm_gate_bwd"] = {"bound": "hbm", "achieved": a_, "peak": hbm_peak, "unit": "GB/s",
                                          "frac": a_ / hbm_peak, "algorithmic_bytes_per_launch": lnb_bytes,
                                          "ms": kern_ms[H.PROFILE_NORM_BWD]}
            cpy = same_size_copy_gbs(lnb_bytes)
            rooflines["norm_gate_bwd"]["same_size_copy"] = {
                "achieved": cpy, "unit": "GB/s", "frac": a_ / cpy,
                "what": "torch device copy of the same bytes from cold memory, CUDA events"}
            # table gradients: every (pair, head) dX^T tile (fp16) and every pair's u8 bucket tile read
            rooflines["table_gradients"] = hbm_line(
                H.PROFILE_TABLE_GRAD, n_pairs * (wl.H * 32768 + 16384),
                f"{n_pairs} pairs x {wl.H} heads of 32 KB dX^T + 16 KB buckets read")
            # dZ assembly: dQ fp32 and Z_Q fp16 read, dZ_Q fp16 written, dZ_U, dZ_V, dZ_K fp16 read back for
            # db1 (the db2 / dgamma / dbeta finishes read a few partial rows more)
            rooflines["dz_assembly"] = hbm_line(H.PROFILE_DZ, 14 * T * D, "14 bytes per token and feature")
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_oracle_sample(wl, backward)
        h2d = int((h_x.numel() + h_dy.numel()) * 2 + h_off.numel() * 8 + h_ts.numel() * 8)
        d2h = int(h_y.numel() * 2 + ((h_dx.numel() * 2 + h_grads.numel() * 4) if backward else 0))
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOADS[args.workload]["desc"], "global_batch": wl.B * world,
                       "tokens_per_rank": T, "seq_len": "jagged", "parallelism": f"dp{world}",
                       "rank_cost_imbalance": float(rank_cost.max() / rank_cost.mean()) if world > 1 else 1.0,
                       "attention_operands": "fp16 U|V|Q|K, P and G, fp32 accumulation and O",
                       "l2": "flushed before every timed step (512 MB written, then 256 MB read)"},
            "roofline": {"bound": "tensor", "kernel": "attn_fwd_persistent_kernel (jagged pointwise attention forward)",
                         "achieved": achieved, "peak": tf_peak, "unit": "TFLOP/s", "frac": achieved / tf_peak,
                         "peak_kind": f"{peak_kind} bf16 burst (dense)", "traffic": traffic_record(args.workload),
                         "algorithmic_flops_per_launch": flops, "ms": kern_ms[H.PROFILE_ATTN_FWD],
                         "timing": "CUDA events recorded by the library right around the kernel, inside as many "
                                   "timed replays of the step (a graph with those event nodes) as the headline"},
            "rooflines": rooflines,
            "workloads": extra,
            "step_breakdown_ms": {k: float(seg[:, i].mean()) for i, k in enumerate(names)},
            "timing": ("device time of CUDA-graph replays of the whole step" if world == 1 else
                       "device time of eagerly launched steps, gradient all-reduce overlapped on a side stream") +
                      " (events on the launching stream); step_breakdown_ms from eager launches",
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "d2h": "Y" + (", dX and the eight gradients" if backward else ""),
                    "method": f"{n_e2e} steps as one timed region, eager launches through the C ABI; each step's "
                              "host-to-device inputs and device-to-host results cross on two copy streams "
                              "while the neighbouring steps compute (two buffer sets); L2 flushed once before "
                              "the region"},
            "gpu_launches": int((n_fwd_kernels + (n_bwd_kernels if backward else 0)) * args.steps),
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
