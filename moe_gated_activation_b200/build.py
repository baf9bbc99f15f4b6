"""Builds libmoeact.so (the CUDA kernels and their C ABI) in the package
directory for sm_100a with nvcc: every translation unit of csrc/ is compiled
to an object in parallel (the fused kernels are split across several), then
linked.  Run ``python -m moe_gated_activation_b200.build``."""
from __future__ import annotations

import concurrent.futures
import glob
import os
import shutil
import subprocess
import sys
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libmoeact.so")
CSRC = os.path.join(PKG, "csrc")
OBJDIR = os.path.join(PKG, "_build")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC",
    # every rounding is an explicit intrinsic; keep the compiler from fusing
    # any remaining multiply-add, and keep IEEE division and subnormals
    "-fmad=false", "-prec-div=true", "-ftz=false",
]

_lock = threading.Lock()


def units():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def sources():
    return (units() + glob.glob(os.path.join(CSRC, "*.cuh"))
            + [os.path.join(ROOT, "include", "moeact.h")])


def nvcc_path():
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libmoeact")
    return cand


def is_stale():
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in sources())


def _compile(nvcc, src, extra_flags, verbose):
    obj = os.path.join(OBJDIR, os.path.basename(src)[:-3] + f".{os.getpid()}.o")
    cmd = [nvcc, *NVCC_FLAGS, *extra_flags, "-c", "-o", obj, src]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    return obj


def build(force: bool = False, verbose: bool = False, extra_flags=()) -> str:
    with _lock:
        if not force and not is_stale():
            return LIB
        nvcc = nvcc_path()
        os.makedirs(OBJDIR, exist_ok=True)
        jobs = max(1, min(len(units()), os.cpu_count() or 1))
        with concurrent.futures.ThreadPoolExecutor(jobs) as ex:
            objs = list(ex.map(lambda u: _compile(nvcc, u, extra_flags, verbose), units()))
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
        for o in objs:
            os.remove(o)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
