"""Build libgdn.so in-tree with nvcc for sm_100a (B200).

    python -m gated_deltanet_linear_21_b200.build [--verbose]

The library is one translation unit (csrc/gdn_api.cu) that includes every
kernel header, compiled without fast-math (IEEE rounding of the basic
operations) and with line info for the profiler. A second build with
-DGDN_DEBUG, libgdn_debug.so, adds device-side index checks that report
through the device error word instead of faulting (same ABI).
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libgdn.so")
DEBUG_LIB = os.path.join(PKG, "libgdn_debug.so")   # -DGDN_DEBUG: device-side index checks
SOURCES = ["gdn_api.cu"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-I", os.path.join(ROOT, "include"), "-I", CSRC,
]


def _nvcc() -> str:
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    path = os.path.join(cuda, "bin", "nvcc")
    return path if os.path.exists(path) else "nvcc"


def _inputs():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files.append(os.path.join(ROOT, "include", "gdn.h"))
    return files


def up_to_date(lib: str = None) -> bool:
    lib = lib or LIB
    if not os.path.exists(lib):
        return False
    t = os.path.getmtime(lib)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def _build_one(lib: str, extra, force: bool, verbose: bool) -> str:
    if not force and up_to_date(lib):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *NVCC_FLAGS, *extra, *(["-Xptxas", "-v"] if verbose else []), "-o", tmp,
           *[os.path.join(CSRC, s) for s in SOURCES]]
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False, debug: bool = True) -> str:
    """Build libgdn.so and (debug=True) the index-checked libgdn_debug.so; the
    path of libgdn.so is returned."""
    _build_one(LIB, [], force, verbose)
    if debug:
        _build_one(DEBUG_LIB, ["-DGDN_DEBUG"], force, False)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
    print(DEBUG_LIB)
