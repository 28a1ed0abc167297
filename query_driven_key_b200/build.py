"""Build libthink.so (the C-ABI CUDA library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libthink.so")
DEBUG_LIB = os.path.join(PKG, "libthink_debug.so")  # -DTHINK_DEBUG: index checks at the global stores

NVCC_FLAGS = [
    "-O3", "-std=c++17",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo",
    "-Xcompiler", "-fPIC",
    "-Xptxas", "-warn-spills",
    "-shared",
]


def _sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _deps():
    return _sources() + sorted(glob.glob(os.path.join(CSRC, "*.cuh"))) + \
        sorted(glob.glob(os.path.join(INCLUDE, "*.h"))) + [os.path.abspath(__file__)]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _build_one(lib: str, flags, force: bool, verbose: bool) -> str:
    if not force and os.path.exists(lib):
        newest = max(os.path.getmtime(p) for p in _deps())
        if os.path.getmtime(lib) >= newest:
            return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *flags, "-I", INCLUDE, "-I", CSRC, *_sources(), "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False, extra_flags=(), debug: bool = True) -> str:
    """Compile csrc/*.cu into libthink.so next to this file (and the debug
    build libthink_debug.so); skip what is up to date."""
    _build_one(LIB, list(extra_flags), force, verbose)
    if debug:
        _build_one(DEBUG_LIB, ["-DTHINK_DEBUG", *extra_flags], force, verbose)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra_flags=["-Xptxas", "-v"] if "--ptxas-v" in sys.argv else [])
