"""Throughput of the HSTU layer hot path on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c2] [--impl ours|reference]

A step is one pass of the layer (f1+SiLU, jagged attention, LayerNorm-gate, f2+residual) over one
seeded synthetic batch of the named workload, inputs resident in HBM. The L2 is flushed (a 512 MB
write) before every timed step; each step is bracketed by CUDA events on the launching stream and
the summed device time is taken as the max over ranks. Under torchrun every rank processes its own
batch (different seed): weak scaling, no collective on the forward data path.

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
WORKLOAD_DESC = {
    "c2": "HSTU layer forward bf16: B=32 jagged sequences, lengths U[64,1024], d_model 256, H 4, "
          "d_qk=d_v=64, N=1024, seed = rank",
    "c3": "HSTU layer forward bf16: B=8 sequences, lengths Pareto(1.2) clipped to [256,8192], d_model 512, "
          "H 8, d_qk=d_v=64, N=8192, seed = rank",
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """Samples nvidia-smi SM clocks and throttle reasons every 200 ms while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.samples.append(parts)

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        mx = [float(s[2]) for s in self.samples if s[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in self.samples for i in range(4) if s[5 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.samples)}


def attn_flops(offsets: np.ndarray, D: int) -> float:
    """Algorithmic attention forward flops: 2 D sum_b n_b (n_b + 1) (causal pairs only, QK^T and PV)."""
    n = np.diff(offsets).astype(np.float64)
    return float(2.0 * D * np.sum(n * (n + 1)))


def traffic_record(workload: str):
    """ncu DRAM bytes of one attention launch, valid only for the kernel source it was taken on."""
    p = os.path.join(ROOT, "profiles", f"attn_fwd_{workload}.traffic.json")
    src = os.path.join(ROOT, "hstu_sequential_transduction_causal_b200", "csrc", "attn_fwd_sm100.cu")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return rec.get("dram_bytes_per_launch") if rec.get("kernel_sha") == sha else None


def cpu_oracle_sample(wl, budget_s: float = 20.0):
    """Times the oracle layer forward on the first sequences of the workload until ~budget_s."""
    from oracle import hstu_oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:  # noqa: BLE001
        cores = 1
    thr = O.time_bucket_thresholds(128)
    p = wl.layers[0]
    tokens = 0
    seqs = 0
    t0 = time.perf_counter()
    for b in range(wl.B):
        s, e = int(wl.offsets[b]), int(wl.offsets[b + 1])
        off = np.array([0, e - s], np.int64)
        O.layer_fwd(wl.x[s:e], p, off, wl.timestamps[s:e], wl.H, 1.0 / wl.N, wl.pos_max_len, thr)
        tokens += e - s
        seqs += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": tokens / dt, "unit": "tokens/s", "cores": int(cores), "kind": "oracle",
            "sample": f"first {seqs} of {wl.B} sequences ({tokens} tokens), numpy fp64 layer forward, "
                      f"{dt:.1f} s wall"}


def run_reference(args, rank, world):
    from hstu_sequential_transduction_causal_b200 import workloads as W
    if rank != 0:
        return
    wl = W.make_workload(args.workload, seed=0)
    times, toks = [], []
    for i in range(args.warmup + args.steps):
        r = cpu_oracle_sample(wl, budget_s=args.ref_budget)
        if i >= args.warmup:
            toks.append(r["value"])
    value = float(np.median(toks))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD_DESC[args.workload], "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
                             "sample": r["sample"]},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="c2", choices=sorted(WORKLOAD_DESC))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-budget", type=float, default=15.0)
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
    from hstu_sequential_transduction_causal_b200.runtime import DeviceLayer, JaggedBatch, SavedActs, to_dev, workspace

    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if rank == 0:
        build()
    if world > 1:
        dist.barrier()
    H.lib()
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()

    wl = W.make_workload(args.workload, seed=rank)
    bf = True
    D, Hh, T = wl.D, wl.H, wl.T
    jag = JaggedBatch(wl.offsets, wl.timestamps, device=dev)
    layer = DeviceLayer.upload(wl.layers[0], D, Hh, bf, device=dev)
    x = to_dev(wl.x, torch.bfloat16, dev)
    y = torch.empty(T, D, dtype=torch.bfloat16, device=dev)
    sv = SavedActs.empty(T, D, torch.bfloat16, keep_z=False, device=dev)
    adesc = H.make_attn_desc(Hh, D // Hh, D // Hh, 1.0 / wl.N, wl.pos_max_len, H.HSTU_F16, 4 * D, 4 * D, 4 * D, D)
    ws = workspace(H.hstu_attn_workspace_size(adesc, jag.struct), dev)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    n_kernels = {"uvqk": 1, "attn": 2, "norm_gate": 1, "out_proj": 1}

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        H.hstu_uvqk_fwd(T, D, H.HSTU_BF16, H.HSTU_F16, x, D, layer.W1, layer.b1, sv.uvqk, None, ws)
        if ev:
            ev[1].record(stream)
        H.hstu_attn_fwd(adesc, jag.struct, sv.uvqk[:, 2 * D:], sv.uvqk[:, 3 * D:], sv.uvqk[:, D:], layer.rab_pos,
                        layer.rab_time, sv.o, ws)
        if ev:
            ev[2].record(stream)
        H.hstu_norm_gate_fwd(T, D, H.HSTU_F32, H.HSTU_F16, H.HSTU_BF16, sv.o, D, sv.uvqk, 4 * D, layer.gamma, layer.beta, 1e-5, sv.g, sv.mu,
                             sv.rstd)
        if ev:
            ev[3].record(stream)
        H.hstu_out_proj_fwd(T, D, H.HSTU_BF16, sv.g, layer.W2, layer.b2, x, H.HSTU_BF16, y, H.HSTU_BF16, None, ws)
        if ev:
            ev[4].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if H.hstu_sync_status(ws) != 0:
        raise RuntimeError("device status error during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for i in range(args.steps):
            flush.zero_()
            step(evs[i])
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    st = H.hstu_sync_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st} in the timed region")
    seg = np.array([[e[k].elapsed_time(e[k + 1]) for k in range(4)] for e in evs])   # ms
    total_ms = float(seg.sum())
    attn_ms = float(seg[:, 1].mean())
    t_tensor = torch.tensor([total_ms, attn_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t_tensor, op=dist.ReduceOp.MAX)
    total_ms, attn_ms_max = float(t_tensor[0]), float(t_tensor[1])
    tokens_all = float(T) * world          # same-shape batches per rank (seeded per rank)
    if world > 1:
        tt = torch.tensor([float(T)], dtype=torch.float64, device=dev)
        dist.all_reduce(tt)
        tokens_all = float(tt.item())
    value = tokens_all * args.steps / (total_ms / 1e3)

    # end to end through the public layer entry point, host buffers in the timed region
    from hstu_sequential_transduction_causal_b200.runtime import LayerRunner
    run = LayerRunner(layer, jag, 1.0 / wl.N, wl.pos_max_len, torch.bfloat16, torch.bfloat16, device=dev)
    x_host = torch.from_numpy(wl.x).to(torch.bfloat16).pin_memory()
    y_host = torch.empty(T, D, dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty(T, D, dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        x_dev.copy_(x_host, non_blocking=True)
        run.forward(x_dev)
        y_host.copy_(run.y, non_blocking=True)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_ms = 0.0
    for _ in range(args.steps):
        flush.zero_()
        e0.record(stream)
        x_dev.copy_(x_host, non_blocking=True)
        run.forward(x_dev)
        y_host.copy_(run.y, non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        e2e_ms += e0.elapsed_time(e1)
    tt = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    e2e_value = tokens_all * args.steps / (float(tt.item()) / 1e3)

    if rank == 0:
        peaks, peak_kind = load_peaks()
        flops = attn_flops(wl.offsets, D)
        achieved = flops / (attn_ms_max / 1e3) / 1e12
        peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
        traffic = traffic_record(args.workload)
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_oracle_sample(wl)
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD_DESC[args.workload], "global_batch": wl.B * world,
                       "tokens_per_rank": T, "seq_len": "jagged", "parallelism": f"dp{world}",
                       "l2": "flushed (512 MB write) before every timed step"},
            "roofline": {"bound": "tensor", "kernel": "attn_fwd_tc_kernel (+ work list)",
                         "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                         "peak_kind": f"{peak_kind} bf16 sustained", "traffic": traffic,
                         "algorithmic_flops_per_launch": flops},
            "step_breakdown_ms": {k: float(seg[:, i].mean()) for i, k in
                                  enumerate(["uvqk", "attn", "norm_gate", "out_proj"])},
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "tokens/s",
                    "h2d_bytes_per_step": int(x_host.numel() * 2), "d2h_bytes_per_step": int(y_host.numel() * 2)},
            "gpu_launches": int(sum(n_kernels.values()) * args.steps),
            "clocks": clk.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
