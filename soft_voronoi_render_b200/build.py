"""Build libsad.so (the C-ABI CUDA library) in-tree for sm_100a."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OUT_DIR = os.path.join(HERE, "_build")
LIB = os.path.join(OUT_DIR, "libsad.so")
# the debug build: the same kernels with device-side bounds checks that count
# refused accesses in the statistics block (-DSAD_CHECKS)
LIB_CHECKS = os.path.join(OUT_DIR, "libsad_checks.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
    "--expt-relaxed-constexpr",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))) + \
        [os.path.join(ROOT, "include", "sad.h")]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _build_one(lib: str, extra: list, force: bool, verbose_ptxas: bool) -> str:
    if not force and os.path.exists(lib):
        t = os.path.getmtime(lib)
        if all(os.path.getmtime(f) <= t for f in _inputs()):
            return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc()] + NVCC_FLAGS + extra + (["-Xptxas", "-v"] if verbose_ptxas else []) + \
        ["-I", os.path.join(ROOT, "include"), "-shared", "-o", tmp] + sources()
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose_ptxas: bool = False, checks: bool = True) -> str:
    """Build libsad.so (and, with checks, the bounds-checked libsad_checks.so);
    returns the path of libsad.so."""
    os.makedirs(OUT_DIR, exist_ok=True)
    _build_one(LIB, [], force, verbose_ptxas)
    if checks:
        _build_one(LIB_CHECKS, ["-DSAD_CHECKS"], force, False)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))
