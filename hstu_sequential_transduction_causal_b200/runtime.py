"""Host-side orchestration around the C ABI: device buffers, workspaces, descriptors.

Nothing here computes: it uploads seeded inputs, allocates the caller-owned buffers the library
writes into (via torch, which owns device memory and streams), fills the descriptors and calls
the binding. Every arithmetic step runs inside libhstu.so.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

from . import hstu as H


def to_dev(a: np.ndarray, dtype: torch.dtype, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device=device, dtype=dtype)


@dataclass
class DeviceLayer:
    """One layer's parameters on the GPU in the layout the library expects."""
    D: int
    H: int
    dtype_code: int
    W1: torch.Tensor
    b1: torch.Tensor
    W2: torch.Tensor
    b2: torch.Tensor
    gamma: torch.Tensor
    beta: torch.Tensor
    rab_pos: torch.Tensor
    rab_time: torch.Tensor

    @classmethod
    def upload(cls, p, D: int, H_: int, bf16: bool, device="cuda") -> "DeviceLayer":
        wdt = torch.bfloat16 if bf16 else torch.float32
        f32 = torch.float32
        return cls(D=D, H=H_, dtype_code=H.HSTU_BF16 if bf16 else H.HSTU_F32,
                   W1=to_dev(p.W1, wdt, device), b1=to_dev(p.b1, f32, device), W2=to_dev(p.W2, wdt, device),
                   b2=to_dev(p.b2, f32, device), gamma=to_dev(p.gamma, f32, device),
                   beta=to_dev(p.beta, f32, device), rab_pos=to_dev(p.rab_pos, f32, device),
                   rab_time=to_dev(p.rab_time, f32, device))

    def weights(self) -> H.hstu_layer_weights_t:
        return H.layer_weights(self.W1, self.b1, self.W2, self.b2, self.gamma, self.beta, self.rab_pos,
                               self.rab_time)


@dataclass
class SavedActs:
    uvqk: torch.Tensor
    z: Optional[torch.Tensor]
    o: torch.Tensor
    g: torch.Tensor
    mu: torch.Tensor
    rstd: torch.Tensor
    attn_bias: Optional[torch.Tensor] = None   # the backward's bias tiles, written by the forward

    @classmethod
    def empty(cls, T: int, D: int, dtype: torch.dtype, keep_z: bool, device="cuda",
              bias_cache_bytes: int = 0) -> "SavedActs":
        act = torch.float16 if dtype == torch.bfloat16 else dtype     # U|V|Q|K, Z and G in fp16
        return cls(uvqk=torch.empty(T, 4 * D, dtype=act, device=device),
                   z=torch.empty(T, 4 * D, dtype=act, device=device) if keep_z else None,
                   o=torch.empty(T, D, dtype=torch.float32, device=device),
                   g=torch.empty(T, D, dtype=act, device=device),
                   mu=torch.empty(T, dtype=torch.float32, device=device),
                   rstd=torch.empty(T, dtype=torch.float32, device=device),
                   attn_bias=(torch.empty(bias_cache_bytes, dtype=torch.uint8, device=device)
                              if bias_cache_bytes > 0 else None))

    def struct(self) -> H.hstu_layer_saved_t:
        return H.layer_saved(self.uvqk, self.z, self.o, self.g, self.mu, self.rstd, self.attn_bias)


class JaggedBatch:
    """Offsets and timestamps on the GPU plus the host-side sizes the descriptors need."""

    def __init__(self, offsets: np.ndarray, timestamps: np.ndarray, max_len: Optional[int] = None,
                 device="cuda"):
        self.offsets_np = np.asarray(offsets, np.int64)
        self.B = int(self.offsets_np.shape[0] - 1)
        self.T = int(self.offsets_np[-1])
        lens = np.diff(self.offsets_np)
        self.max_len = int(max_len if max_len is not None else (lens.max() if self.B else 0))
        self.offsets = to_dev(self.offsets_np, torch.int64, device)
        self.timestamps = to_dev(np.asarray(timestamps, np.int64), torch.int64, device)
        self.struct = H.make_jagged(self.offsets, self.timestamps, self.max_len)


def shard_rows(offsets: np.ndarray, rank_of: np.ndarray, rank: int):
    """The sequences a data-parallel split (hstu_dp_partition) gives `rank`, in batch order: their
    offsets (int64 [B_r + 1], starting at 0) and the global rows they own (int64 [T_r]), for
    gathering x, dy and timestamps of the rank's shard from the global batch."""
    offsets = np.asarray(offsets, np.int64)
    mine = np.nonzero(np.asarray(rank_of) == rank)[0]
    lens = offsets[mine + 1] - offsets[mine]
    off = np.zeros(mine.shape[0] + 1, np.int64)
    np.cumsum(lens, out=off[1:])
    rows = (np.concatenate([np.arange(offsets[b], offsets[b + 1], dtype=np.int64) for b in mine])
            if mine.size else np.zeros(0, np.int64))
    return off, rows


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A zero-filled workspace (its first word is the device status word)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


class LayerRunner:
    """Runs ``hstu_layer_fwd`` for one layer on a fixed jagged batch with reusable buffers."""

    def __init__(self, layer: DeviceLayer, jag: JaggedBatch, inv_N: float, pos_max_len: int,
                 x_dtype: torch.dtype, y_dtype: torch.dtype, keep_z: bool = False, device="cuda",
                 bias_cache: Optional[bool] = None):
        """keep_z: a backward follows (Z is kept); bias_cache (default: keep_z in BF16 mode): the forward
        also writes the backward's attention bias tiles into saved.attn_bias."""
        self.layer, self.jag = layer, jag
        cdt = torch.bfloat16 if layer.dtype_code == H.HSTU_BF16 else torch.float32
        code = {torch.bfloat16: H.HSTU_BF16, torch.float32: H.HSTU_F32}
        self.desc = H.make_layer_desc(layer.D, layer.H, inv_N, pos_max_len, layer.dtype_code, code[x_dtype],
                                      code[y_dtype])
        if bias_cache is None:
            bias_cache = keep_z and layer.dtype_code == H.HSTU_BF16
        nbias = H.hstu_layer_bias_cache_size(self.desc, jag.struct) if bias_cache else 0
        self.saved = SavedActs.empty(jag.T, layer.D, cdt, keep_z, device, nbias)
        self.saved_struct = self.saved.struct()
        self.ws = workspace(H.hstu_layer_workspace_size(self.desc, jag.struct), device)
        self.y = torch.empty(jag.T, layer.D, dtype=y_dtype, device=device)
        self.weights = layer.weights()

    def forward(self, x: torch.Tensor, x_f16: Optional[torch.Tensor] = None,
                y_f16: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        H.hstu_layer_fwd(self.desc, self.jag.struct, self.weights, x, x_f16, self.y, y_f16,
                         self.saved_struct, self.ws, stream)
        return self.y

    def device_status(self) -> int:
        return H.hstu_sync_status(self.ws)


class Encoder:
    """A stack of HSTU layers on an fp32 residual stream (BF16 compute).

    forward() keeps each layer's input and saved activations; backward() runs the layers in reverse
    and returns dX of the stack, leaving each layer's parameter gradients in ``grads[l]``. Every
    step is one hstu_layer_fwd / hstu_layer_bwd call; layer l hands layer l+1 the fp16 copy of its
    output (the next f1 operand) and, going back, the fp16 copy of its dX (the next dy operand).
    """

    def __init__(self, layers, jag: JaggedBatch, inv_N: float, pos_max_len: int, device="cuda"):
        self.layers, self.jag = list(layers), jag
        L, D, T = len(self.layers), self.layers[0].D, jag.T
        self.desc = H.make_layer_desc(D, self.layers[0].H, inv_N, pos_max_len, H.HSTU_BF16, H.HSTU_F32, H.HSTU_F32)
        self.weights = [lay.weights() for lay in self.layers]
        nbias = H.hstu_layer_bias_cache_size(self.desc, jag.struct)
        self.saved = [SavedActs.empty(T, D, torch.bfloat16, True, device, nbias) for _ in range(L)]
        self.saved_structs = [sv.struct() for sv in self.saved]
        self.xs = [None] + [torch.empty(T, D, dtype=torch.float32, device=device) for _ in range(L - 1)]
        self.x16 = [None] + [torch.empty(T, D, dtype=torch.float16, device=device) for _ in range(L - 1)]
        self.y = torch.empty(T, D, dtype=torch.float32, device=device)
        self.dx = [torch.empty(T, D, dtype=torch.float32, device=device) for _ in range(2)]
        self.dx16 = [torch.empty(T, D, dtype=torch.float16, device=device) for _ in range(2)]
        self.ws = workspace(max(H.hstu_layer_workspace_size(self.desc, jag.struct),
                                H.hstu_layer_bwd_workspace_size(self.desc, jag.struct)), device)
        # one flat fp32 row per layer, every view starting on a 16-byte boundary (the weight
        # gradients are accumulated with 16-byte vector atomics)
        sizes = [4 * D * D, 4 * D, D * D, D, D, D, 2 * pos_max_len - 1, 128]
        padded = [(n_ + 3) // 4 * 4 for n_ in sizes]
        self.grad_flat = torch.zeros(L, sum(padded), dtype=torch.float32, device=device)
        self.grads = []
        for l in range(L):
            views, o = [], 0
            for n_, pn in zip(sizes, padded):
                views.append(self.grad_flat[l, o:o + n_])
                o += pn
            self.grads.append(views)
        self.grad_structs = [H.layer_grads(*g) for g in self.grads]

    def forward(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        """x: fp32 [T, D] (kept by reference until backward)."""
        self.xs[0] = x
        L = len(self.layers)
        for l in range(L):
            last = l == L - 1
            y = self.y if last else self.xs[l + 1]
            H.hstu_layer_fwd(self.desc, self.jag.struct, self.weights[l], self.xs[l], self.x16[l], y,
                             None if last else self.x16[l + 1], self.saved_structs[l], self.ws, stream)
        return self.y

    def backward(self, dy: torch.Tensor, stream=None) -> torch.Tensor:
        g, g16 = dy, None
        for l in reversed(range(len(self.layers))):
            dx, dx16 = self.dx[l & 1], self.dx16[l & 1]
            H.hstu_layer_bwd(self.desc, self.jag.struct, self.weights[l], self.xs[l], self.x16[l],
                             self.saved_structs[l], g, g16, dx, dx16 if l > 0 else None, self.grad_structs[l],
                             self.ws, stream)
            g, g16 = dx, dx16
        return g

    def device_status(self) -> int:
        return H.hstu_sync_status(self.ws)


def stochastic_length(raw: JaggedBatch, keys: torch.Tensor, alpha: float, x: Optional[torch.Tensor] = None,
                      device="cuda"):
    """Subsamples a raw jagged batch on the GPU. Returns (JaggedBatch of the kept tokens, kept raw
    indices, kept rows of x or None). One host read of the kept-token count sizes the outputs."""
    ws = workspace(256, device)
    new_off = torch.empty(raw.B + 1, dtype=torch.int64, device=device)
    H.hstu_stochastic_length_offsets(raw.struct, alpha, new_off, ws)
    off_host = new_off.cpu().numpy()
    if H.hstu_sync_status(ws) != 0:
        raise RuntimeError("malformed raw offsets")
    T2 = int(off_host[-1])
    kept = torch.empty(max(T2, 1), dtype=torch.int64, device=device)
    ts = torch.empty(max(T2, 1), dtype=torch.int64, device=device)
    x_out = None
    code = None
    if x is not None:
        x_out = torch.empty(max(T2, 1), x.shape[1], dtype=x.dtype, device=device)
        code = H._dtype_code(x)
    H.hstu_stochastic_length_select(raw.struct, keys, new_off, x, code if code is not None else 0,
                                    x.shape[1] if x is not None else 0, kept, x_out, ts, ws)
    if H.hstu_sync_status(ws) != 0:
        raise RuntimeError("stochastic length selection reported an error")
    lens = np.diff(off_host)
    jag = JaggedBatch.__new__(JaggedBatch)
    jag.offsets_np, jag.B, jag.T = off_host, raw.B, T2
    jag.max_len = int(lens.max()) if raw.B else 0
    jag.offsets, jag.timestamps = new_off, ts[:T2]
    jag.struct = H.make_jagged(jag.offsets, jag.timestamps, jag.max_len)
    return jag, kept[:T2], (x_out[:T2] if x_out is not None else None)
