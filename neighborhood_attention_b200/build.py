"""Build the CUDA library ``libna.so`` in-tree with nvcc for sm_100a.

    python neighborhood_attention_b200/build.py [--force] [-v]

Run it by path (or load it with ``load_builder()`` from ``__graft_entry__``):
importing the package itself requires the built library.

The CUDA runtime is linked statically; the tensor-map encoder is reached
through cudaGetDriverEntryPoint, so the library needs no -lcuda.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libna.so")
SOURCES = ["na_api.cu", "na_fwd_simt.cu", "na_fwd_gather.cu", "na_fwd_sm100.cu", "na_bwd_simt.cu",
           "na_bwd_sm100.cu"]
HEADERS = ["na_internal.h", "na_sched.cuh", "na_stages.cuh", "na_ptx.cuh"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "na.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared",
           "-Xptxas", "-v" if verbose else "-O3", "-I", os.path.join(ROOT, "include"),
           "-o", tmp] + [os.path.join(CSRC, f) for f in SOURCES]
    subprocess.check_call(cmd, cwd=PKG)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
