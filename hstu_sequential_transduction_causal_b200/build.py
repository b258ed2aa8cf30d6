"""Builds libhstu.so in-tree with nvcc for sm_100a.

    python -m hstu_sequential_transduction_causal_b200.build [--force] [--ptxas-verbose] [--debug]

Each translation unit under csrc/ is compiled to an object in csrc/_build/ (in parallel), then
linked into csrc/libhstu.so against the CUDA runtime. Rebuilds only when a source or header is
newer than the library. --debug builds csrc/libhstu_debug.so (objects in csrc/_build_debug/) with
-DHSTU_DEBUG: every checked index (HSTU_DCHECK: table gathers, output rows) records HSTU_ERR_DEVICE
in the status word and skips the access. The binding loads it when HSTU_DEBUG=1 is set.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(CSRC, "libhstu.so")
BUILD_DIR = os.path.join(CSRC, "_build")
LIB_DEBUG = os.path.join(CSRC, "libhstu_debug.so")
BUILD_DIR_DEBUG = os.path.join(CSRC, "_build_debug")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
         "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return (_sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
            + glob.glob(os.path.join(INCLUDE, "*.h")))


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _deps())


def _compile(src: str, ptxas_verbose: bool, debug: bool = False) -> str:
    obj = os.path.join(BUILD_DIR_DEBUG if debug else BUILD_DIR, os.path.basename(src)[:-3] + ".o")
    cmd = [NVCC, *ARCH, *FLAGS, *(["-DHSTU_DEBUG"] if debug else []), "-c", src, "-o", obj]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr}")
    if ptxas_verbose and r.stderr:
        sys.stderr.write(r.stderr)
    return obj


def build(force: bool = False, ptxas_verbose: bool = False, debug: bool = False) -> str:
    """Compiles the CUDA library if needed and returns the path of libhstu.so (libhstu_debug.so with
    debug=True)."""
    lib = LIB_DEBUG if debug else LIB
    if not force and not ptxas_verbose and not _stale(lib):
        return lib
    os.makedirs(BUILD_DIR_DEBUG if debug else BUILD_DIR, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, ptxas_verbose, debug), _sources()))
    tmp = lib + ".tmp"
    cmd = [NVCC, *ARCH, "-shared", "--cudart", "static", "-o", tmp, *objs]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    ap.add_argument("--debug", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, ptxas_verbose=a.ptxas_verbose, debug=a.debug))
