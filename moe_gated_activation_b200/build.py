"""Builds libmoeact.so (the CUDA kernels and their C ABI) in the package
directory for sm_100a with nvcc.  Run ``python -m moe_gated_activation_b200.build``."""
from __future__ import annotations

import glob
import os
import shutil
import subprocess
import sys
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libmoeact.so")
MAIN = os.path.join(PKG, "csrc", "capi.cu")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC",
    # every rounding is an explicit intrinsic; keep the compiler from fusing
    # any remaining multiply-add, and keep IEEE division and subnormals
    "-fmad=false", "-prec-div=true", "-ftz=false",
]

_lock = threading.Lock()


def sources():
    return (glob.glob(os.path.join(PKG, "csrc", "*.cu"))
            + glob.glob(os.path.join(PKG, "csrc", "*.cuh"))
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


def build(force: bool = False, verbose: bool = False, extra_flags=()) -> str:
    with _lock:
        if not force and not is_stale():
            return LIB
        tmp = LIB + f".tmp{os.getpid()}"
        cmd = [nvcc_path(), *NVCC_FLAGS, *extra_flags, "-o", tmp, MAIN]
        if verbose:
            print(" ".join(cmd), file=sys.stderr)
        subprocess.run(cmd, check=True)
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
