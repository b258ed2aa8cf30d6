"""Seeded synthetic workloads for the HSTU layer.

This module draws random numbers and lays them out in the shapes the layer consumes. It holds
none of the layer's arithmetic: the CUDA path (through the binding) and the CPU oracle (in the
tests) both take its arrays as inputs, so the two sides always see bit-identical inputs.

Shapes and distributions follow the five workloads the library is measured on:

* ``c1`` one fp32 layer over four sequences of lengths {17, 64, 100, 256}, d_model 64, 2 heads;
* ``c2`` one bf16 layer, 32 sequences with lengths uniform in [64, 1024], d_model 256, 4 heads;
* ``c3`` one bf16 layer forward+backward, 8 sequences with Pareto(1.2) lengths clipped to
  [256, 8192], d_model 512, 8 heads;
* ``c4`` an 8-layer bf16 stack forward+backward, 64 raw sequences with lengths uniform in
  [512, 4096] that are subsampled by Stochastic Length, d_model 512, 8 heads, fp32 residual;
* ``c5`` M-FALCON ranking: 16 users with 2048-token prefixes, 4 layers, 1024 candidates per user
  scored in micro-batches of 256.

Common recipe: X ~ N(0, 1); weights ~ N(0, std 1/sqrt(fan_in)); biases 0; the relative-position
and relative-time tables ~ N(0, std 0.02); LayerNorm gamma = 1, beta = 0; timestamps are int64
seconds starting at 1,700,000,000 with gaps floor(Exp(mean 3600)) (so equal timestamps occur).
In bf16 workloads every floating input is rounded to bf16 once, here, so both sides consume the
same representable values.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np

T0 = 1_700_000_000
GAP_MEAN_S = 3600.0
N_TIME_BUCKETS = 128
TABLE_STD = 0.02

CONFIGS: Dict[str, dict] = {
    "c1": dict(lengths=[17, 64, 100, 256], D=64, H=2, dtype="f32", N=256, pos_max_len=256,
               layers=1, backward=False),
    "c2": dict(B=32, len_lo=64, len_hi=1024, D=256, H=4, dtype="bf16", N=1024,
               pos_max_len=1024, layers=1, backward=False),
    "c3": dict(B=8, pareto_alpha=1.2, len_lo=256, len_hi=8192, D=512, H=8, dtype="bf16",
               N=8192, pos_max_len=8192, layers=1, backward=True),
    "c4": dict(B=64, len_lo=512, len_hi=4096, sl_alpha=1.6, D=512, H=8, dtype="bf16",
               N=4096, pos_max_len=4096, layers=8, backward=True),
    "c5": dict(users=16, prefix=2048, m=1024, b_m=256, D=512, H=8, dtype="bf16", N=2049,
               pos_max_len=2049, layers=4, backward=False),
}


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round to the nearest bf16 value (ties to even); returns float32 holding bf16 values."""
    a32 = np.ascontiguousarray(a, dtype=np.float32)
    u = a32.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    out = r.astype(np.uint32).view(np.float32)
    # NaN/inf are not produced by these generators; keep them out explicitly.
    assert np.all(np.isfinite(out)), "bf16 rounding overflowed"
    return out


@dataclass
class LayerParams:
    W1: np.ndarray        # [4D, D] projection to U|V|Q|K
    b1: np.ndarray        # [4D]
    W2: np.ndarray        # [D, D] output projection
    b2: np.ndarray        # [D]
    gamma: np.ndarray     # [D]
    beta: np.ndarray      # [D]
    rab_pos: np.ndarray   # [2*pos_max_len - 1]
    rab_time: np.ndarray  # [N_TIME_BUCKETS]


@dataclass
class Workload:
    name: str
    D: int
    H: int
    dtype: str                 # "f32" or "bf16"
    N: float                   # attention normaliser
    pos_max_len: int
    offsets: np.ndarray        # int64 [B+1]
    timestamps: np.ndarray     # int64 [T]
    x: np.ndarray              # float32 [T, D]
    layers: List[LayerParams]
    dy: Optional[np.ndarray] = None   # float32 [T, D] upstream gradient (backward workloads)
    extra: dict = field(default_factory=dict)

    @property
    def T(self) -> int:
        return int(self.offsets[-1])

    @property
    def B(self) -> int:
        return int(self.offsets.shape[0] - 1)

    @property
    def lengths(self) -> np.ndarray:
        return np.diff(self.offsets)

    @property
    def max_len(self) -> int:
        return int(self.lengths.max()) if self.B > 0 else 0


def offsets_from_lengths(lengths) -> np.ndarray:
    lengths = np.asarray(lengths, dtype=np.int64)
    off = np.zeros(lengths.shape[0] + 1, dtype=np.int64)
    np.cumsum(lengths, out=off[1:])
    return off


def draw_timestamps(rng: np.random.Generator, lengths) -> np.ndarray:
    """Per sequence: t_0 = T0, later tokens add floor(Exp(mean 3600 s)) second gaps."""
    parts = []
    for n in lengths:
        n = int(n)
        gaps = np.floor(rng.exponential(GAP_MEAN_S, size=max(n - 1, 0))).astype(np.int64)
        t = np.empty(n, dtype=np.int64)
        if n:
            t[0] = T0
            np.cumsum(gaps, out=t[1:])
            t[1:] += T0
        parts.append(t)
    return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)


def draw_layer(rng: np.random.Generator, D: int, pos_max_len: int, bf16: bool) -> LayerParams:
    W1 = rng.standard_normal((4 * D, D)) / np.sqrt(D)
    W2 = rng.standard_normal((D, D)) / np.sqrt(D)
    rab_pos = rng.standard_normal(2 * pos_max_len - 1) * TABLE_STD
    rab_time = rng.standard_normal(N_TIME_BUCKETS) * TABLE_STD
    cast = round_bf16 if bf16 else (lambda a: np.asarray(a, dtype=np.float32))
    return LayerParams(
        W1=cast(W1), b1=np.zeros(4 * D, np.float32), W2=cast(W2), b2=np.zeros(D, np.float32),
        gamma=np.ones(D, np.float32), beta=np.zeros(D, np.float32),
        rab_pos=cast(rab_pos), rab_time=cast(rab_time))


def _draw_lengths(rng: np.random.Generator, cfg: dict) -> np.ndarray:
    if "lengths" in cfg:
        return np.asarray(cfg["lengths"], dtype=np.int64)
    if "pareto_alpha" in cfg:
        u = 1.0 - rng.random(cfg["B"])          # (0, 1]
        n = np.floor(cfg["len_lo"] * u ** (-1.0 / cfg["pareto_alpha"]))
        return np.clip(n, cfg["len_lo"], cfg["len_hi"]).astype(np.int64)
    return rng.integers(cfg["len_lo"], cfg["len_hi"] + 1, size=cfg["B"]).astype(np.int64)


def make_workload(name: str, seed: int = 0, *, lengths=None, D=None, H=None, dtype=None,
                  N=None, pos_max_len=None, layers=None, backward=None, B=None) -> Workload:
    """Draw one of the named workloads (``c1``..``c4``), optionally overriding its shape.

    ``c4`` returns the *raw* sequences plus the Stochastic Length random keys in
    ``extra["sl_keys"]`` (int64, one per raw token) and ``extra["sl_alpha"]``; the subsampling
    itself is part of the method and happens in the library / the oracle.
    """
    cfg = dict(CONFIGS[name])
    for k, v in dict(lengths=lengths, D=D, H=H, dtype=dtype, N=N, pos_max_len=pos_max_len,
                     layers=layers, backward=backward, B=B).items():
        if v is not None:
            cfg[k] = v
    rng = np.random.default_rng(seed)
    lens = _draw_lengths(rng, cfg)
    off = offsets_from_lengths(lens)
    ts = draw_timestamps(rng, lens)
    bf16 = cfg["dtype"] == "bf16"
    T = int(off[-1])
    x = rng.standard_normal((T, cfg["D"]))
    x = round_bf16(x) if bf16 else x.astype(np.float32)
    layer_list = [draw_layer(rng, cfg["D"], cfg["pos_max_len"], bf16)
                  for _ in range(cfg.get("layers", 1))]
    dy = None
    if cfg.get("backward"):
        dy = rng.standard_normal((T, cfg["D"]))
        dy = round_bf16(dy) if bf16 else dy.astype(np.float32)
    wl = Workload(name=name, D=cfg["D"], H=cfg["H"], dtype=cfg["dtype"], N=float(cfg["N"]),
                  pos_max_len=cfg["pos_max_len"], offsets=off, timestamps=ts, x=x,
                  layers=layer_list, dy=dy)
    if "sl_alpha" in cfg:
        wl.extra["sl_alpha"] = cfg["sl_alpha"]
        wl.extra["sl_keys"] = rng.integers(0, 2 ** 62, size=T, dtype=np.int64)
    return wl


@dataclass
class FalconWorkload:
    D: int
    H: int
    N: float
    pos_max_len: int
    layers: List[LayerParams]
    prefix_offsets: np.ndarray    # int64 [users+1]
    prefix_ts: np.ndarray         # int64 [users*prefix]
    prefix_x: np.ndarray          # float32 [users*prefix, D]
    cand_x: np.ndarray            # float32 [users*m, D]
    request_ts: np.ndarray        # int64 [users] (every candidate of a user carries it)
    m: int
    b_m: int

    @property
    def users(self) -> int:
        return int(self.prefix_offsets.shape[0] - 1)


def make_falcon_workload(seed: int = 0, *, users=None, prefix=None, m=None, b_m=None,
                         D=None, H=None, layers=None, N=None, pos_max_len=None,
                         prefix_lengths=None) -> FalconWorkload:
    cfg = dict(CONFIGS["c5"])
    for k, v in dict(users=users, prefix=prefix, m=m, b_m=b_m, D=D, H=H, layers=layers, N=N,
                     pos_max_len=pos_max_len).items():
        if v is not None:
            cfg[k] = v
    rng = np.random.default_rng(seed)
    U, n, D = cfg["users"], cfg["prefix"], cfg["D"]
    if prefix_lengths is not None:      # ragged prefixes (tests); users follows the list
        lens = np.asarray(prefix_lengths, dtype=np.int64)
        U = cfg["users"] = len(lens)
    else:
        lens = np.full(U, n, dtype=np.int64)
    off = offsets_from_lengths(lens)
    ts = draw_timestamps(rng, lens)
    last = np.array([ts[off[u + 1] - 1] if lens[u] > 0 else T0 for u in range(U)], dtype=np.int64)
    req = last + np.floor(rng.exponential(GAP_MEAN_S, size=U)).astype(np.int64)
    px = round_bf16(rng.standard_normal((int(off[-1]), D)))
    cx = round_bf16(rng.standard_normal((U * cfg["m"], D)))
    layer_list = [draw_layer(rng, D, cfg["pos_max_len"], True) for _ in range(cfg["layers"])]
    return FalconWorkload(D=D, H=cfg["H"], N=float(cfg["N"]), pos_max_len=cfg["pos_max_len"],
                          layers=layer_list, prefix_offsets=off, prefix_ts=ts, prefix_x=px,
                          cand_x=cx, request_ts=req, m=cfg["m"], b_m=cfg["b_m"])
