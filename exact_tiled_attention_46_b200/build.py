"""Builds the CUDA library libfa46.so in-tree for sm_100a with nvcc.

    python -m exact_tiled_attention_46_b200.build [--verbose] [--force] [--debug]

--debug builds libfa46_debug.so instead (FA_DEBUG: every global store checks its
index and reports a failure through the device status instead of writing).

The library is one translation unit (csrc/fa_api.cu) that includes every
kernel; it links the CUDA runtime statically and reaches the driver's
tensor-map encoder through the runtime's entry-point query, so it needs no
libcuda at link time.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libfa46.so")
DEBUG_LIB = os.path.join(PKG, "libfa46_debug.so")   # FA_DEBUG: index checks on every global store
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources():
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cu", ".cuh")))


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + [os.path.join(ROOT, "include", "fa.h")]
    return any(os.path.getmtime(s) > t for s in deps)


def build(verbose: bool = False, force: bool = False, debug: bool = False) -> str:
    lib = DEBUG_LIB if debug else LIB
    if not force and not needs_build(lib):
        return lib
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I" + os.path.join(ROOT, "include"), "-I" + CSRC,
           "-o", lib + ".tmp", os.path.join(CSRC, "fa_api.cu")]
    if debug:
        cmd.insert(1, "-DFA_DEBUG")
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force="--force" in sys.argv, debug="--debug" in sys.argv))
