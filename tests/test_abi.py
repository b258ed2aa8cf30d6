"""CPU checks of the C ABI boundary: the library loads, exports every function the header
declares, and the binding's signature table matches the header's argument counts."""
import ctypes
import os
import re

import pytest
import torch

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


# These two hand fake, never dereferenced device addresses to calls that the host must reject; they
# run only where no GPU is visible, so a missed check can never pass a fake address to a kernel.
cpu_only = pytest.mark.skipif(torch.cuda.is_available(), reason="fake device addresses")


@cpu_only
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


@cpu_only
def test_layer_bwd_rejects_misaligned_gradients_on_host(lib):
    """dW1 / dW2 are accumulated with 16-byte vector atomics: a pointer off that boundary is refused
    (HSTU_ERR_UNSUPPORTED) before anything reaches the GPU."""
    Hb._lib = None
    L = Hb.lib()
    D, T = 256, 300
    jag = Hb.hstu_jagged_t(B=1, max_len=T, T=T, offsets=1 << 20, timestamps=2 << 20)
    desc = Hb.make_layer_desc(D, 4, 1.0 / 512, 512, Hb.HSTU_BF16, Hb.HSTU_BF16, Hb.HSTU_BF16)
    need = L.hstu_layer_bwd_workspace_size(ctypes.byref(desc), ctypes.byref(jag))
    w = Hb.hstu_layer_weights_t(*[(i + 3) << 20 for i in range(8)])
    saved = Hb.hstu_layer_saved_t(*[(i + 20) << 20 for i in range(6)])
    good = [(i + 40) << 20 for i in range(8)]
    bad = list(good)
    bad[0] += 4                                    # dW1 4 bytes off a 16-byte boundary
    r = L.hstu_layer_bwd(ctypes.byref(desc), ctypes.byref(jag), ctypes.byref(w), 60 << 20, None, ctypes.byref(saved),
                         61 << 20, None, 62 << 20, None, ctypes.byref(Hb.hstu_layer_grads_t(*bad)), 63 << 20, need,
                         None)
    assert r == 2


def test_header_compiles_as_c_and_links(lib, tmp_path):
    """The boundary is usable from plain C: a C99 program that includes only include/hstu.h builds
    with -Wall -Werror, links against libhstu.so and makes the calls that need no GPU."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_hstu.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "hstu.h"

int main(void) {
  if (hstu_abi_version() != HSTU_ABI_VERSION) return 1;
  if (strcmp(hstu_status_string(HSTU_ERR_WORKSPACE), "HSTU_ERR_WORKSPACE") != 0) return 2;
  hstu_jagged_t jag;
  memset(&jag, 0, sizeof jag);
  jag.B = -1;                                       /* malformed: refused on the host */
  if (hstu_worklist_capacity(&jag) != -1) return 3;
  hstu_attn_desc_t desc;
  memset(&desc, 0, sizeof desc);
  if (hstu_attn_fwd(&desc, &jag, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL) != HSTU_ERR_INVALID_ARG)
    return 4;
  int32_t st = 0;
  if (hstu_sync_status(NULL, NULL, &st) != HSTU_ERR_INVALID_ARG) return 5;
  printf("ok\n");
  return 0;
}
''')
    exe = tmp_path / "use_hstu"
    libdir = os.path.dirname(B.LIB)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           str(src), "-o", str(exe), f"-L{libdir}", "-lhstu", f"-Wl,-rpath,{libdir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)
