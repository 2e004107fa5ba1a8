"""Builds libkivi.so (the C ABI of include/kivi.h) in-tree for sm_100a with nvcc."""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libkivi.so")
DEBUG_LIB = os.path.join(PKG, "libkivi_debug.so")
# debug build: short bounded waits (about 1 ms), copy bounds checks, a test hook
DEBUG_FLAGS = ["-DKIVI_DEBUG_BUILD", "-DKIVI_DEBUG_BOUNDS", "-DKIVI_DEBUG_WAIT_CYCLES=2000000LL"]
SOURCES = ["kivi_api.cu", "kivi_quant.cu", "kivi_attn.cu", "kivi_bf16_attn.cu",
           "kivi_prefill_attn.cu"]
NVCC_FLAGS = [
    "-O3", "-std=c++17",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-warn-spills",
]


def _inputs():
    files = [os.path.join(CSRC, f) for f in os.listdir(CSRC)
             if f.endswith((".cu", ".cuh", ".h"))]
    return files + [os.path.join(ROOT, "include", "kivi.h")]


def stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Builds libkivi.so (or, with debug=True, libkivi_debug.so) when stale."""
    lib = DEBUG_LIB if debug else LIB
    if not force and not stale(lib):
        return lib
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = lib + ".tmp"
    cmd = [nvcc, *NVCC_FLAGS, *(DEBUG_FLAGS if debug else []), "-o", tmp,
           *[os.path.join(CSRC, s) for s in SOURCES]]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, debug="--debug" in sys.argv))
