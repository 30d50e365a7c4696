"""Build libtern.so (CUDA, sm_100a) in-tree with nvcc.

The library is a plain C-ABI shared object: include/tern.h declares its entry
points.  cudart is linked statically so the .so loads on machines without a
GPU (argument checks then still work; any CUDA call reports an error).

build(debug=True) writes libtern_debug.so instead: the same sources compiled
with -DTERN_DEBUG_GUARDS, whose decode-step kernels check their shared-memory
and global indices, count failed checks in a device word (the access is
skipped, nothing traps) and report them through tern_sync_status as
TERN_ERR_GUARD.  It stands in for a memory checker on machines where none
can run; the product binding loads libtern.so only.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libtern.so")
LIB_DEBUG = os.path.join(PKG, "libtern_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + [os.path.join(INCLUDE, "tern.h")]


def up_to_date(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(p) <= t for p in _deps())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    lib = LIB_DEBUG if debug else LIB
    if not force and up_to_date(lib):
        return lib
    tmp = lib + ".tmp"
    cmd = [NVCC, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
           "-cudart", "static", "-I", INCLUDE, "-I", CSRC, *sources(), "-o", tmp]
    if debug:
        cmd.insert(1, "-DTERN_DEBUG_GUARDS")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building libtern.so")
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
