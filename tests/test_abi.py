"""CPU checks of the C ABI boundary: the library loads, exports every function the header
declares, and the binding's signature table matches the header's argument counts."""
import ctypes
import os
import re

import pytest

from hstu_sequential_transduction_causal_b200 import build as B
from hstu_sequential_transduction_causal_b200 import hstu as Hb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hstu.h")


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    decls = {}
    for m in re.finditer(r"\b([a-z_0-9]+\s*\*?)\s+(hstu_[a-z_0-9]+)\s*\(([^)]*)\)\s*;", text):
        args = m.group(3).strip()
        n = 0 if args in ("", "void") else args.count(",") + 1
        decls[m.group(2)] = n
    return decls


@pytest.fixture(scope="module")
def lib():
    B.build()
    return ctypes.CDLL(B.LIB)


def test_header_declares_the_boundary():
    fns = header_functions()
    for name in ("hstu_layer_fwd", "hstu_attn_fwd", "hstu_uvqk_fwd", "hstu_norm_gate_fwd",
                 "hstu_out_proj_fwd", "hstu_jagged_worklist", "hstu_time_buckets", "hstu_sync_status"):
        assert name in fns
    text = open(HEADER).read()
    assert "torch" not in text.lower().replace("pytorch", "")
    assert 'extern "C"' in text


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), f"{name} missing from libhstu.so"


def test_binding_signatures_match_header():
    fns = header_functions()
    assert set(Hb.SIGNATURES) == set(fns), set(Hb.SIGNATURES) ^ set(fns)
    for name, n in fns.items():
        assert len(Hb.SIGNATURES[name][1]) == n, name


def test_abi_version_and_status_strings(lib):
    lib.hstu_abi_version.restype = ctypes.c_int32
    assert lib.hstu_abi_version() == 1
    lib.hstu_status_string.restype = ctypes.c_char_p
    lib.hstu_status_string.argtypes = [ctypes.c_int32]
    assert lib.hstu_status_string(0) == b"HSTU_OK"
    assert lib.hstu_status_string(5) == b"HSTU_ERR_TIMEOUT"


def test_host_validation_without_gpu(lib):
    """Argument errors are caught on the host before any CUDA call."""
    Hb._lib = None
    L = Hb.lib()
    jag = Hb.hstu_jagged_t(B=-1, max_len=0, T=0, offsets=None, timestamps=None)
    assert L.hstu_worklist_capacity(ctypes.byref(jag)) == -1
    desc = Hb.make_attn_desc(2, 32, 32, 1.0, 8, Hb.HSTU_BF16, 128, 128, 128, 64)
    jag = Hb.hstu_jagged_t(B=1, max_len=4, T=4, offsets=1024, timestamps=2048)
    # bf16 needs d = 64
    r = L.hstu_attn_fwd(ctypes.byref(desc), ctypes.byref(jag), 4096, 4096, 4096, 4096, 4096, 4096, 4096, 1 << 20,
                        None)
    assert r == 2
    desc = Hb.make_attn_desc(2, 64, 64, 1.0, 8, Hb.HSTU_BF16, 128, 128, 128, 128)
    r = L.hstu_attn_fwd(ctypes.byref(desc), ctypes.byref(jag), 4096, 4096, 4096, 4096, 4096, 4096, 4096, 16, None)
    assert r == 3   # workspace too small
    desc.n_time_buckets = 129
    r = L.hstu_attn_fwd(ctypes.byref(desc), ctypes.byref(jag), 4096, 4096, 4096, 4096, 4096, 4096, 4096, 1 << 20,
                        None)
    assert r == 2
