"""Build the CUDA library in-tree: bit_kv_cache_24_b200/libnvfp4.so (sm_100a only), and its
bounds-checked debug build libnvfp4_checked.so (NVFP4_DEBUG_CHECKS: every index-computed device
access is checked against its buffer's extent and skipped with NVFP4_ERR_OUT_OF_BOUNDS in the
status word instead of faulting; select it at run time with NVFP4_LIB=<path>).

    python -m bit_kv_cache_24_b200.build [--force] [--checked]

nvcc compiles every csrc/*.cu for sm_100a (no PTX fallback for other GPUs) into one shared
library with a static CUDA runtime, so the library loads without a GPU (it only needs the driver
at the first CUDA call).  No fast-math: every rounding that decides a code is explicit.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(os.path.dirname(HERE), "include")
LIB = os.path.join(HERE, "libnvfp4.so")
CHECKED_LIB = os.path.join(HERE, "libnvfp4_checked.so")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-Xptxas", "-warn-spills",
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        sorted(glob.glob(os.path.join(CSRC, "*.h"))) + sorted(glob.glob(os.path.join(INCLUDE, "*.h")))


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _deps())


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    lib = CHECKED_LIB if checked else LIB
    if not force and not needs_build(lib):
        return lib
    tmp = lib + ".tmp"
    extra = ["-DNVFP4_DEBUG_CHECKS"] if checked else []
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", INCLUDE, "-shared", "-o", tmp, *_sources()]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True, checked="--checked" in sys.argv)
