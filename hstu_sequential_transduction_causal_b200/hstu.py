"""ctypes binding of libhstu.so: the C ABI's entry points under the same names.

Argument marshalling only: descriptors become ctypes structures, torch tensors become device
pointers, the current torch CUDA stream becomes the cudaStream_t. Every step of the computation
runs in the library's CUDA kernels; nothing here computes. If the library is missing, every
call raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from .build import LIB as _LIB_RELEASE, LIB_DEBUG as _LIB_DEBUG

# HSTU_DEBUG=1 selects the checked-index build (build.py --debug)
_LIB_PATH = _LIB_DEBUG if os.environ.get("HSTU_DEBUG", "0") not in ("", "0") else _LIB_RELEASE

c_i32, c_i64, c_f32, c_vp, c_sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t

HSTU_F32, HSTU_BF16, HSTU_F16 = 0, 1, 2
(HSTU_OK, HSTU_ERR_INVALID_ARG, HSTU_ERR_UNSUPPORTED, HSTU_ERR_WORKSPACE, HSTU_ERR_CUDA, HSTU_ERR_TIMEOUT,
 HSTU_ERR_DEVICE) = range(7)
STATUS = {0: "HSTU_OK", 1: "HSTU_ERR_INVALID_ARG", 2: "HSTU_ERR_UNSUPPORTED", 3: "HSTU_ERR_WORKSPACE",
          4: "HSTU_ERR_CUDA", 5: "HSTU_ERR_TIMEOUT", 6: "HSTU_ERR_DEVICE"}


class HstuError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        extra = ""
        if code == 4 and _lib is not None:
            extra = f" (cudaError {_lib.hstu_last_cuda_error()})"
        super().__init__(f"{fn} returned {STATUS.get(code, code)}{extra}")


class hstu_jagged_t(ctypes.Structure):
    _fields_ = [("B", c_i32), ("max_len", c_i32), ("T", c_i64), ("offsets", c_vp), ("timestamps", c_vp)]


class hstu_attn_desc_t(ctypes.Structure):
    _fields_ = [("H", c_i32), ("d_qk", c_i32), ("d_v", c_i32), ("inv_N", c_f32), ("pos_max_len", c_i32),
                ("n_time_buckets", c_i32), ("dtype", c_i32), ("o_dtype", c_i32), ("ld_q", c_i64), ("ld_k", c_i64),
                ("ld_v", c_i64), ("ld_o", c_i64)]


class hstu_layer_desc_t(ctypes.Structure):
    _fields_ = [("D", c_i32), ("H", c_i32), ("inv_N", c_f32), ("pos_max_len", c_i32),
                ("n_time_buckets", c_i32), ("ln_eps", c_f32), ("dtype", c_i32), ("x_dtype", c_i32),
                ("y_dtype", c_i32)]


class hstu_layer_weights_t(ctypes.Structure):
    _fields_ = [(n, c_vp) for n in ("W1", "b1", "W2", "b2", "gamma", "beta", "rab_pos", "rab_time")]


class hstu_layer_saved_t(ctypes.Structure):
    _fields_ = [(n, c_vp) for n in ("uvqk", "z", "o", "g", "mu", "rstd", "attn_bias")]


class hstu_layer_grads_t(ctypes.Structure):
    _fields_ = [(n, c_vp) for n in ("dW1", "db1", "dW2", "db2", "dgamma", "dbeta", "drab_pos", "drab_time")]


class hstu_falcon_desc_t(ctypes.Structure):
    _fields_ = [("L", c_i32), ("users", c_i32), ("m", c_i32), ("b_m", c_i32), ("D", c_i32), ("H", c_i32),
                ("inv_N", c_f32), ("pos_max_len", c_i32), ("n_time_buckets", c_i32), ("ln_eps", c_f32)]


class hstu_rab_ext_t(ctypes.Structure):
    _fields_ = [("per_head", c_i32), ("n_types", c_i32), ("token_type", c_vp), ("rab_type", c_vp)]


class hstu_norm_in_t(ctypes.Structure):
    _fields_ = [("gamma", c_vp), ("beta", c_vp), ("xn", c_vp), ("mu", c_vp), ("rstd", c_vp), ("dgamma", c_vp),
                ("dbeta", c_vp)]


P = ctypes.POINTER
# name -> (restype, argtypes); the list every test checks against include/hstu.h
SIGNATURES = {
    "hstu_abi_version": (c_i32, []),
    "hstu_status_string": (ctypes.c_char_p, [c_i32]),
    "hstu_last_cuda_error": (c_i32, []),
    "hstu_sync_status": (c_i32, [c_vp, c_vp, P(c_i32)]),
    "hstu_set_wait_limit": (None, [ctypes.c_uint64]),
    "hstu_debug_timeout_probe": (c_i32, [c_vp, c_sz, c_vp]),
    "hstu_profile_events": (c_i32, [c_i32, c_vp, c_vp]),
    "hstu_dp_sequence_cost": (ctypes.c_double, [c_i64, c_i32]),
    "hstu_dp_partition": (c_i32, [c_vp, c_i32, c_i32, c_i32, c_vp, c_vp]),
    "hstu_layer_bwd_ready_events": (c_i32, [c_vp, c_vp]),
    "hstu_worklist_capacity": (c_i64, [P(hstu_jagged_t)]),
    "hstu_jagged_worklist": (c_i32, [P(hstu_jagged_t), c_vp, c_vp, c_vp]),
    "hstu_time_buckets": (c_i32, [P(hstu_jagged_t), c_i32, c_vp, c_vp, c_vp]),
    "hstu_uvqk_fwd": (c_i32, [c_i64, c_i32, c_i32, c_i32, c_vp, c_i64, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "hstu_attn_workspace_size": (c_sz, [P(hstu_attn_desc_t), P(hstu_jagged_t)]),
    "hstu_attn_fwd": (c_i32, [P(hstu_attn_desc_t), P(hstu_jagged_t), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                              c_vp, c_sz, c_vp]),
    "hstu_attn_bwd_workspace_size": (c_sz, [P(hstu_attn_desc_t), P(hstu_jagged_t)]),
    "hstu_attn_bwd": (c_i32, [P(hstu_attn_desc_t), P(hstu_jagged_t), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                              c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "hstu_linear_bf16": (c_i32, [c_i64, c_i64, c_i64, c_vp, c_i64, c_i32, c_vp, c_i64, c_i32, c_vp, c_vp, c_i32,
                                 c_i64, c_vp, c_i32, c_i64, c_i32, c_vp, c_sz, c_vp]),
    "hstu_layer_bwd_workspace_size": (c_sz, [P(hstu_layer_desc_t), P(hstu_jagged_t)]),
    "hstu_layer_bias_cache_size": (c_sz, [P(hstu_layer_desc_t), P(hstu_jagged_t)]),
    "hstu_layer_bwd": (c_i32, [P(hstu_layer_desc_t), P(hstu_jagged_t), P(hstu_layer_weights_t), c_vp, c_vp,
                               P(hstu_layer_saved_t), c_vp, c_vp, c_vp, c_vp, P(hstu_layer_grads_t), c_vp, c_sz,
                               c_vp]),
    "hstu_attn_ext_workspace_size": (c_sz, [P(hstu_attn_desc_t), P(hstu_jagged_t), P(hstu_rab_ext_t)]),
    "hstu_attn_fwd_ext": (c_i32, [P(hstu_attn_desc_t), P(hstu_jagged_t), P(hstu_rab_ext_t), c_vp, c_vp, c_vp, c_vp,
                                  c_vp, c_vp, c_vp, c_sz, c_vp]),
    "hstu_attn_bwd_ext_workspace_size": (c_sz, [P(hstu_attn_desc_t), P(hstu_jagged_t), P(hstu_rab_ext_t)]),
    "hstu_attn_bwd_ext": (c_i32, [P(hstu_attn_desc_t), P(hstu_jagged_t), P(hstu_rab_ext_t), c_vp, c_vp, c_vp, c_vp,
                                  c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "hstu_attn_fwd_noalloc": (c_i32, [P(hstu_attn_desc_t), P(hstu_jagged_t), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                                      c_vp]),
    "hstu_attn_fwd_noalloc_status": (c_i32, [c_vp, P(c_i32)]),
    "hstu_norm_gate_fwd": (c_i32, [c_i64, c_i32, c_i32, c_i32, c_i32, c_vp, c_i64, c_vp, c_i64, c_vp, c_vp,
                                   c_f32, c_vp, c_vp, c_vp, c_vp]),
    "hstu_out_proj_workspace_size": (c_sz, [c_i32, c_i32]),
    "hstu_out_proj_fwd": (c_i32, [c_i64, c_i32, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_i32, c_vp, c_i32, c_vp,
                                  c_vp, c_sz, c_vp]),
    "hstu_layer_workspace_size": (c_sz, [P(hstu_layer_desc_t), P(hstu_jagged_t)]),
    "hstu_layer_fwd": (c_i32, [P(hstu_layer_desc_t), P(hstu_jagged_t), P(hstu_layer_weights_t), c_vp, c_vp,
                               c_vp, c_vp, P(hstu_layer_saved_t), c_vp, c_sz, c_vp]),
    "hstu_stochastic_length_offsets": (c_i32, [P(hstu_jagged_t), ctypes.c_double, c_vp, c_vp, c_sz, c_vp]),
    "hstu_stochastic_length_select": (c_i32, [P(hstu_jagged_t), c_vp, c_vp, c_vp, c_i32, c_i32, c_vp, c_vp, c_vp,
                                              c_vp, c_sz, c_vp]),
    "hstu_falcon_cache_size": (c_sz, [P(hstu_falcon_desc_t), P(hstu_jagged_t)]),
    "hstu_falcon_workspace_size": (c_sz, [P(hstu_falcon_desc_t), P(hstu_jagged_t)]),
    "hstu_layer_norm_in_workspace_size": (c_sz, [P(hstu_layer_desc_t), P(hstu_jagged_t)]),
    "hstu_layer_fwd_norm_in": (c_i32, [P(hstu_layer_desc_t), P(hstu_jagged_t), P(hstu_layer_weights_t),
                                       P(hstu_norm_in_t), c_vp, c_vp, c_vp, P(hstu_layer_saved_t), c_vp, c_sz, c_vp]),
    "hstu_layer_bwd_norm_in": (c_i32, [P(hstu_layer_desc_t), P(hstu_jagged_t), P(hstu_layer_weights_t),
                                       P(hstu_norm_in_t), c_vp, P(hstu_layer_saved_t), c_vp, c_vp, c_vp,
                                       P(hstu_layer_grads_t), c_vp, c_sz, c_vp]),
    "hstu_falcon_append_workspace_size": (c_sz, [P(hstu_falcon_desc_t), P(hstu_jagged_t), P(hstu_jagged_t),
                                                  P(hstu_jagged_t)]),
    "hstu_falcon_append": (c_i32, [P(hstu_falcon_desc_t), P(hstu_layer_weights_t), P(hstu_jagged_t), c_vp,
                                   P(hstu_jagged_t), c_vp, P(hstu_jagged_t), c_vp, c_vp, c_vp, c_sz, c_vp]),
    "hstu_falcon_fwd": (c_i32, [P(hstu_falcon_desc_t), P(hstu_layer_weights_t), P(hstu_jagged_t), c_vp, c_vp, c_i32,
                                c_vp, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
}

_lib: Optional[ctypes.CDLL] = None


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """Loads libhstu.so (libhstu_debug.so under HSTU_DEBUG=1; built in-tree by ``build.py``); raises if
    it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"libhstu.so not built ({_LIB_PATH}); run "
                               "`python -m hstu_sequential_transduction_causal_b200.build`")
        l = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


# ----------------------------------------------------------------------------------------------
# marshalling helpers
# ----------------------------------------------------------------------------------------------

def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    return t.data_ptr()


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return HSTU_BF16
    if t.dtype == torch.float32:
        return HSTU_F32
    if t.dtype == torch.float16:
        return HSTU_F16
    raise ValueError(f"unsupported dtype {t.dtype}")


def _check(fn: str, code: int):
    if code != 0:
        raise HstuError(fn, code)


def make_jagged(offsets: torch.Tensor, timestamps: torch.Tensor, max_len: int) -> hstu_jagged_t:
    """offsets: int64 [B+1] on the GPU; timestamps: int64 [T] on the GPU; T is read from the
    caller's host knowledge of the batch (``timestamps.shape[0]``), never from the device."""
    assert offsets.dtype == torch.int64 and timestamps.dtype == torch.int64
    return hstu_jagged_t(B=offsets.shape[0] - 1, max_len=int(max_len), T=timestamps.shape[0],
                         offsets=_ptr(offsets), timestamps=_ptr(timestamps) if timestamps.numel() else None)


def make_attn_desc(H, d_qk, d_v, inv_N, pos_max_len, dtype_code, ld_q, ld_k, ld_v, ld_o,
                   n_time_buckets=128, o_dtype_code=HSTU_F32) -> hstu_attn_desc_t:
    return hstu_attn_desc_t(H=H, d_qk=d_qk, d_v=d_v, inv_N=inv_N, pos_max_len=pos_max_len,
                            n_time_buckets=n_time_buckets, dtype=dtype_code, o_dtype=o_dtype_code, ld_q=ld_q,
                            ld_k=ld_k, ld_v=ld_v, ld_o=ld_o)


def make_layer_desc(D, H, inv_N, pos_max_len, dtype_code, x_dtype_code, y_dtype_code,
                    n_time_buckets=128, ln_eps=1e-5) -> hstu_layer_desc_t:
    return hstu_layer_desc_t(D=D, H=H, inv_N=inv_N, pos_max_len=pos_max_len, n_time_buckets=n_time_buckets,
                             ln_eps=ln_eps, dtype=dtype_code, x_dtype=x_dtype_code, y_dtype=y_dtype_code)


# ----------------------------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ----------------------------------------------------------------------------------------------

def hstu_abi_version() -> int:
    return lib().hstu_abi_version()


def hstu_status_string(code: int) -> str:
    return lib().hstu_status_string(code).decode()


def hstu_sync_status(ws: torch.Tensor, stream=None) -> int:
    out = c_i32(0)
    _check("hstu_sync_status", lib().hstu_sync_status(_ptr(ws), _stream(stream), ctypes.byref(out)))
    return out.value


def hstu_set_wait_limit(cycles: int) -> None:
    lib().hstu_set_wait_limit(int(cycles))


PROFILE_ATTN_FWD, PROFILE_ATTN_BWD, PROFILE_NORM_FWD, PROFILE_NORM_BWD = 0, 1, 2, 3
PROFILE_BIAS, PROFILE_TABLE_GRAD, PROFILE_DZ = 4, 5, 6


def hstu_profile_events(kernel: int, start=None, stop=None) -> None:
    """Records the two torch.cuda.Event objects (timing enabled) around the given kernel of later
    calls on this host thread; no events disables. The events are recorded once first so that
    their CUDA handles exist."""
    if start is None or stop is None:
        _check("hstu_profile_events", lib().hstu_profile_events(kernel, None, None))
        return
    for ev in (start, stop):
        ev.record()
    _check("hstu_profile_events", lib().hstu_profile_events(kernel, ctypes.c_void_p(start.cuda_event),
                                                            ctypes.c_void_p(stop.cuda_event)))


def hstu_dp_partition(lengths, D: int, world: int):
    """(rank of each sequence int32 [B], cost of each rank float64 [world]) of the library's
    cost-balanced split of one global batch (host arrays; no GPU needed)."""
    import numpy as np
    lens = np.ascontiguousarray(lengths, dtype=np.int64)
    rank_of = np.zeros(lens.shape[0], dtype=np.int32)
    cost = np.zeros(world, dtype=np.float64)
    _check("hstu_dp_partition", lib().hstu_dp_partition(lens.ctypes.data, lens.shape[0], D, world,
                                                        rank_of.ctypes.data, cost.ctypes.data))
    return rank_of, cost


def hstu_layer_bwd_ready_events(early=None, w1=None) -> None:
    """torch.cuda.Event objects recorded by later hstu_layer_bwd calls on this thread when their
    early gradients (dW2, db2, dgamma, dbeta, tables) and then dW1, db1 are final; none disables."""
    if early is None or w1 is None:
        _check("hstu_layer_bwd_ready_events", lib().hstu_layer_bwd_ready_events(None, None))
        return
    for ev in (early, w1):
        ev.record()
    _check("hstu_layer_bwd_ready_events", lib().hstu_layer_bwd_ready_events(ctypes.c_void_p(early.cuda_event),
                                                                            ctypes.c_void_p(w1.cuda_event)))


def hstu_debug_timeout_probe(ws: torch.Tensor, stream=None) -> None:
    _check("hstu_debug_timeout_probe", lib().hstu_debug_timeout_probe(_ptr(ws), ws.numel() * ws.element_size(),
                                                                      _stream(stream)))


def hstu_worklist_capacity(jag: hstu_jagged_t) -> int:
    return lib().hstu_worklist_capacity(ctypes.byref(jag))


def hstu_jagged_worklist(jag: hstu_jagged_t, items: torch.Tensor, count: torch.Tensor, stream=None) -> None:
    _check("hstu_jagged_worklist", lib().hstu_jagged_worklist(ctypes.byref(jag), _ptr(items), _ptr(count),
                                                              _stream(stream)))


def hstu_time_buckets(jag: hstu_jagged_t, n_buckets: int, sq_offsets: torch.Tensor, out: torch.Tensor,
                      stream=None) -> None:
    _check("hstu_time_buckets", lib().hstu_time_buckets(ctypes.byref(jag), n_buckets, _ptr(sq_offsets),
                                                        _ptr(out), _stream(stream)))


def hstu_uvqk_fwd(T, D, dtype_code, act_dtype_code, x, ld_x, W1, b1, uvqk, z, ws, stream=None) -> None:
    _check("hstu_uvqk_fwd", lib().hstu_uvqk_fwd(T, D, dtype_code, act_dtype_code, _ptr(x), ld_x, _ptr(W1), _ptr(b1),
                                                _ptr(uvqk),
                                                _ptr(z), _ptr(ws), ws.numel() * ws.element_size(),
                                                _stream(stream)))


def hstu_attn_workspace_size(desc: hstu_attn_desc_t, jag: hstu_jagged_t) -> int:
    return lib().hstu_attn_workspace_size(ctypes.byref(desc), ctypes.byref(jag))


def hstu_attn_fwd(desc, jag, q, k, v, rab_pos, rab_time, out, ws, stream=None) -> None:
    _check("hstu_attn_fwd", lib().hstu_attn_fwd(ctypes.byref(desc), ctypes.byref(jag), _ptr(q), _ptr(k), _ptr(v),
                                                _ptr(rab_pos), _ptr(rab_time), _ptr(out), _ptr(ws),
                                                ws.numel() * ws.element_size(), _stream(stream)))


def hstu_attn_bwd_workspace_size(desc: hstu_attn_desc_t, jag: hstu_jagged_t) -> int:
    return lib().hstu_attn_bwd_workspace_size(ctypes.byref(desc), ctypes.byref(jag))


def hstu_attn_bwd(desc, jag, q, k, v, d_out, rab_pos, rab_time, dq, dk, dv, d_rab_pos, d_rab_time, ws,
                  stream=None) -> None:
    _check("hstu_attn_bwd", lib().hstu_attn_bwd(ctypes.byref(desc), ctypes.byref(jag), _ptr(q), _ptr(k), _ptr(v),
                                                _ptr(d_out), _ptr(rab_pos), _ptr(rab_time), _ptr(dq), _ptr(dk),
                                                _ptr(dv), _ptr(d_rab_pos), _ptr(d_rab_time), _ptr(ws),
                                                ws.numel() * ws.element_size(), _stream(stream)))


def make_rab_ext(per_head: bool, n_types: int = 0, token_type=None, rab_type=None) -> hstu_rab_ext_t:
    return hstu_rab_ext_t(per_head=int(per_head), n_types=n_types, token_type=_ptr(token_type),
                          rab_type=_ptr(rab_type))


def hstu_attn_ext_workspace_size(desc, jag, ext) -> int:
    return lib().hstu_attn_ext_workspace_size(ctypes.byref(desc), ctypes.byref(jag), ctypes.byref(ext))


def hstu_attn_fwd_ext(desc, jag, ext, q, k, v, rab_pos, rab_time, out, ws, stream=None) -> None:
    _check("hstu_attn_fwd_ext", lib().hstu_attn_fwd_ext(ctypes.byref(desc), ctypes.byref(jag), ctypes.byref(ext),
                                                        _ptr(q), _ptr(k), _ptr(v), _ptr(rab_pos), _ptr(rab_time),
                                                        _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                                                        _stream(stream)))


def hstu_attn_bwd_ext_workspace_size(desc, jag, ext) -> int:
    return lib().hstu_attn_bwd_ext_workspace_size(ctypes.byref(desc), ctypes.byref(jag), ctypes.byref(ext))


def hstu_attn_bwd_ext(desc, jag, ext, q, k, v, d_out, rab_pos, rab_time, dq, dk, dv, d_rab_pos, d_rab_time,
                      d_rab_type, ws, stream=None) -> None:
    _check("hstu_attn_bwd_ext", lib().hstu_attn_bwd_ext(ctypes.byref(desc), ctypes.byref(jag), ctypes.byref(ext),
                                                        _ptr(q), _ptr(k), _ptr(v), _ptr(d_out), _ptr(rab_pos),
                                                        _ptr(rab_time), _ptr(dq), _ptr(dk), _ptr(dv),
                                                        _ptr(d_rab_pos), _ptr(d_rab_time), _ptr(d_rab_type),
                                                        _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def hstu_attn_fwd_noalloc(desc, jag, q, k, v, rab_pos, rab_time, out, stream=None) -> None:
    """hstu_attn_fwd without a workspace: the scratch is a fixed array inside the library (for
    callers that cannot allocate device memory); calls that overlap on the GPU race."""
    _check("hstu_attn_fwd_noalloc", lib().hstu_attn_fwd_noalloc(ctypes.byref(desc), ctypes.byref(jag), _ptr(q), _ptr(k),
                                                                _ptr(v), _ptr(rab_pos), _ptr(rab_time), _ptr(out),
                                                                _stream(stream)))


def hstu_attn_fwd_noalloc_status(stream=None) -> int:
    """Device status of the last hstu_attn_fwd_noalloc call on this device (read and reset)."""
    out = c_i32(0)
    _check("hstu_attn_fwd_noalloc_status", lib().hstu_attn_fwd_noalloc_status(_stream(stream), ctypes.byref(out)))
    return out.value


def hstu_norm_gate_fwd(T, D, o_dtype_code, u_dtype_code, g_dtype_code, o, ld_o, u, ld_u, gamma, beta, eps, g, mu,
                       rstd, stream=None) -> None:
    _check("hstu_norm_gate_fwd", lib().hstu_norm_gate_fwd(T, D, o_dtype_code, u_dtype_code, g_dtype_code, _ptr(o),
                                                          ld_o, _ptr(u), ld_u,
                                                          _ptr(gamma), _ptr(beta), eps, _ptr(g), _ptr(mu),
                                                          _ptr(rstd), _stream(stream)))


def hstu_out_proj_workspace_size(D: int, g_dtype_code: int) -> int:
    return lib().hstu_out_proj_workspace_size(D, g_dtype_code)


def hstu_out_proj_fwd(T, D, dtype_code, g_dtype_code, g, W2, b2, x, x_dtype_code, y, y_dtype_code, y_f16, ws,
                      stream=None) -> None:
    _check("hstu_out_proj_fwd", lib().hstu_out_proj_fwd(T, D, dtype_code, g_dtype_code, _ptr(g), _ptr(W2), _ptr(b2),
                                                        _ptr(x), x_dtype_code, _ptr(y), y_dtype_code, _ptr(y_f16),
                                                        _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def hstu_layer_workspace_size(desc: hstu_layer_desc_t, jag: hstu_jagged_t) -> int:
    return lib().hstu_layer_workspace_size(ctypes.byref(desc), ctypes.byref(jag))


def hstu_layer_fwd(desc, jag, weights: hstu_layer_weights_t, x, x_f16, y, y_f16, saved: hstu_layer_saved_t,
                   ws, stream=None) -> None:
    _check("hstu_layer_fwd", lib().hstu_layer_fwd(ctypes.byref(desc), ctypes.byref(jag), ctypes.byref(weights),
                                                  _ptr(x), _ptr(x_f16), _ptr(y), _ptr(y_f16),
                                                  ctypes.byref(saved), _ptr(ws), ws.numel() * ws.element_size(),
                                                  _stream(stream)))


def layer_weights(W1, b1, W2, b2, gamma, beta, rab_pos, rab_time) -> hstu_layer_weights_t:
    return hstu_layer_weights_t(*[_ptr(t) for t in (W1, b1, W2, b2, gamma, beta, rab_pos, rab_time)])


def layer_saved(uvqk, z, o, g, mu, rstd, attn_bias=None) -> hstu_layer_saved_t:
    return hstu_layer_saved_t(*[_ptr(t) for t in (uvqk, z, o, g, mu, rstd, attn_bias)])


def hstu_linear_bf16(M, N, K, A, lda, a_mn, B, ldb, b_mn, bias, resid, resid_dtype_code, ld_resid, out,
                     out_dtype_code, ld_out, accumulate, ws, stream=None) -> None:
    _check("hstu_linear_bf16", lib().hstu_linear_bf16(M, N, K, _ptr(A), lda, int(a_mn), _ptr(B), ldb, int(b_mn),
                                                      _ptr(bias), _ptr(resid), resid_dtype_code, ld_resid, _ptr(out),
                                                      out_dtype_code, ld_out, int(accumulate), _ptr(ws),
                                                      ws.numel() * ws.element_size(), _stream(stream)))


def hstu_layer_bwd_workspace_size(desc: hstu_layer_desc_t, jag: hstu_jagged_t) -> int:
    return lib().hstu_layer_bwd_workspace_size(ctypes.byref(desc), ctypes.byref(jag))


def hstu_layer_bias_cache_size(desc: hstu_layer_desc_t, jag: hstu_jagged_t) -> int:
    return lib().hstu_layer_bias_cache_size(ctypes.byref(desc), ctypes.byref(jag))


def hstu_layer_bwd(desc, jag, weights: hstu_layer_weights_t, x, x_f16, saved: hstu_layer_saved_t, dy, dy_f16, dx,
                   dx_f16, grads: hstu_layer_grads_t, ws, stream=None) -> None:
    _check("hstu_layer_bwd", lib().hstu_layer_bwd(ctypes.byref(desc), ctypes.byref(jag), ctypes.byref(weights),
                                                  _ptr(x), _ptr(x_f16), ctypes.byref(saved), _ptr(dy),
                                                  _ptr(dy_f16), _ptr(dx), _ptr(dx_f16), ctypes.byref(grads),
                                                  _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def layer_grads(dW1, db1, dW2, db2, dgamma, dbeta, drab_pos, drab_time) -> hstu_layer_grads_t:
    return hstu_layer_grads_t(*[_ptr(t) for t in (dW1, db1, dW2, db2, dgamma, dbeta, drab_pos, drab_time)])


def make_falcon_desc(L, users, m, b_m, D, H, inv_N, pos_max_len, n_time_buckets=128,
                     ln_eps=1e-5) -> hstu_falcon_desc_t:
    return hstu_falcon_desc_t(L, users, m, b_m, D, H, inv_N, pos_max_len, n_time_buckets, ln_eps)


def hstu_falcon_cache_size(desc: hstu_falcon_desc_t, prefix: hstu_jagged_t) -> int:
    return lib().hstu_falcon_cache_size(ctypes.byref(desc), ctypes.byref(prefix))


def hstu_falcon_workspace_size(desc: hstu_falcon_desc_t, prefix: hstu_jagged_t) -> int:
    return lib().hstu_falcon_workspace_size(ctypes.byref(desc), ctypes.byref(prefix))


def hstu_falcon_fwd(desc: hstu_falcon_desc_t, layers, prefix: hstu_jagged_t, prefix_x, kv_cache, cache_valid,
                    prefix_out, cand_x, request_ts, out, ws, stream=None) -> None:
    """layers: a sequence of hstu_layer_weights_t (marshalled into the host array the call reads)."""
    arr = (hstu_layer_weights_t * len(layers))(*layers)
    _check("hstu_falcon_fwd", lib().hstu_falcon_fwd(ctypes.byref(desc), arr, ctypes.byref(prefix), _ptr(prefix_x),
                                                    _ptr(kv_cache), int(cache_valid), _ptr(prefix_out),
                                                    _ptr(cand_x), _ptr(request_ts), _ptr(out), _ptr(ws),
                                                    ws.numel() * ws.element_size(), _stream(stream)))


def hstu_stochastic_length_offsets(raw: hstu_jagged_t, alpha: float, new_offsets, ws, stream=None) -> None:
    _check("hstu_stochastic_length_offsets",
           lib().hstu_stochastic_length_offsets(ctypes.byref(raw), float(alpha), _ptr(new_offsets), _ptr(ws),
                                                ws.numel() * ws.element_size(), _stream(stream)))


def hstu_stochastic_length_select(raw: hstu_jagged_t, keys, new_offsets, x, x_dtype_code, D, kept, x_out, ts_out, ws,
                                  stream=None) -> None:
    _check("hstu_stochastic_length_select",
           lib().hstu_stochastic_length_select(ctypes.byref(raw), _ptr(keys), _ptr(new_offsets), _ptr(x), x_dtype_code,
                                               D, _ptr(kept), _ptr(x_out), _ptr(ts_out), _ptr(ws),
                                               ws.numel() * ws.element_size(), _stream(stream)))


def hstu_falcon_append_workspace_size(desc, prefix_old, appended, prefix_new) -> int:
    return lib().hstu_falcon_append_workspace_size(ctypes.byref(desc), ctypes.byref(prefix_old), ctypes.byref(appended),
                                                   ctypes.byref(prefix_new))


def hstu_falcon_append(desc, layers, prefix_old, kv_cache_old, appended, app_x, prefix_new, kv_cache_new, app_out,
                       ws, stream=None) -> None:
    """layers: a sequence of hstu_layer_weights_t (marshalled into the host array the call reads)."""
    arr = (hstu_layer_weights_t * len(layers))(*layers)
    _check("hstu_falcon_append", lib().hstu_falcon_append(ctypes.byref(desc), arr, ctypes.byref(prefix_old),
                                                          _ptr(kv_cache_old), ctypes.byref(appended), _ptr(app_x),
                                                          ctypes.byref(prefix_new), _ptr(kv_cache_new),
                                                          _ptr(app_out), _ptr(ws), ws.numel() * ws.element_size(),
                                                          _stream(stream)))


def make_norm_in(gamma, beta, xn, mu, rstd, dgamma=None, dbeta=None) -> hstu_norm_in_t:
    return hstu_norm_in_t(gamma=_ptr(gamma), beta=_ptr(beta), xn=_ptr(xn), mu=_ptr(mu), rstd=_ptr(rstd),
                          dgamma=_ptr(dgamma), dbeta=_ptr(dbeta))


def hstu_layer_norm_in_workspace_size(desc, jag) -> int:
    return lib().hstu_layer_norm_in_workspace_size(ctypes.byref(desc), ctypes.byref(jag))


def hstu_layer_fwd_norm_in(desc, jag, weights, nin, x, y, y_f16, saved, ws, stream=None) -> None:
    _check("hstu_layer_fwd_norm_in", lib().hstu_layer_fwd_norm_in(ctypes.byref(desc), ctypes.byref(jag),
                                                                  ctypes.byref(weights), ctypes.byref(nin), _ptr(x),
                                                                  _ptr(y), _ptr(y_f16), ctypes.byref(saved), _ptr(ws),
                                                                  ws.numel() * ws.element_size(), _stream(stream)))


def hstu_layer_bwd_norm_in(desc, jag, weights, nin, x, saved, dy, dx, dx_f16, grads, ws, stream=None) -> None:
    _check("hstu_layer_bwd_norm_in", lib().hstu_layer_bwd_norm_in(ctypes.byref(desc), ctypes.byref(jag),
                                                                  ctypes.byref(weights), ctypes.byref(nin), _ptr(x),
                                                                  ctypes.byref(saved), _ptr(dy), _ptr(dx),
                                                                  _ptr(dx_f16), ctypes.byref(grads), _ptr(ws),
                                                                  ws.numel() * ws.element_size(), _stream(stream)))
