"""Seeded synthetic inputs (q, k, v ~ N(0, 1)) shared by the oracle side and the
CUDA side of every test and of the benchmark.

This module holds no attention arithmetic.  It only maps (seed, element index)
to a standard-normal sample through a counter-based SplitMix64 generator and a
Box-Muller transform (see ``gen.c``), then rounds to float32, bfloat16 or
float16 (round-to-nearest-even; float16 by numpy's conversion) or OFP8 E4M3
(round-to-nearest-even, saturating at +-448).  Both sides
receive the very same host buffers, so the oracle reads exactly the values
that the GPU receives.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB = os.path.join(_HERE, "libna_gen.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``gen.c`` into ``libna_gen.so`` next to it (gcc, -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            lib.na_gen_normal_f32.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_float,
                                              ctypes.c_void_p, ctypes.c_int]
            lib.na_gen_normal_f32.restype = ctypes.c_int
            lib.na_gen_normal_bf16.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_float,
                                               ctypes.c_void_p, ctypes.c_int]
            lib.na_gen_normal_bf16.restype = ctypes.c_int
            lib.na_gen_normal_e4m3.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_float,
                                               ctypes.c_void_p, ctypes.c_int]
            lib.na_gen_normal_e4m3.restype = ctypes.c_int
            lib.na_gen_round_e4m3.argtypes = [ctypes.c_void_p, ctypes.c_uint64, ctypes.c_void_p]
            lib.na_gen_round_e4m3.restype = None
            lib.na_gen_splitmix64_at.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
            lib.na_gen_splitmix64_at.restype = ctypes.c_uint64
            _lib = lib
    return _lib


def _threads(n: int | None) -> int:
    return int(n) if n else (os.cpu_count() or 1)


def normal_f32(seed: int, shape, scale: float = 1.0, threads: int | None = None) -> np.ndarray:
    """float32 array of N(0, scale^2) samples for stream ``seed``."""
    lib = _load()
    out = np.empty(shape, dtype=np.float32)
    rc = lib.na_gen_normal_f32(seed, out.size, scale, out.ctypes.data, _threads(threads))
    if rc != 0:
        raise RuntimeError("na_gen_normal_f32 failed")
    return out


def normal_bf16_bits(seed: int, shape, scale: float = 1.0, threads: int | None = None) -> np.ndarray:
    """uint16 array holding the bfloat16 (RNE) bit patterns of the same samples."""
    lib = _load()
    out = np.empty(shape, dtype=np.uint16)
    rc = lib.na_gen_normal_bf16(seed, out.size, scale, out.ctypes.data, _threads(threads))
    if rc != 0:
        raise RuntimeError("na_gen_normal_bf16 failed")
    return out


def normal_e4m3_bits(seed: int, shape, scale: float = 1.0, threads: int | None = None) -> np.ndarray:
    """uint8 array holding the OFP8 E4M3 (RNE, saturating at +-448) bit
    patterns of the same samples."""
    lib = _load()
    out = np.empty(shape, dtype=np.uint8)
    rc = lib.na_gen_normal_e4m3(seed, out.size, scale, out.ctypes.data, _threads(threads))
    if rc != 0:
        raise RuntimeError("na_gen_normal_e4m3 failed")
    return out


def round_e4m3_bits(values) -> np.ndarray:
    """E4M3 bit patterns of float32 values (the generator's own rounding)."""
    a = np.ascontiguousarray(np.asarray(values, dtype=np.float32))
    out = np.empty(a.shape, dtype=np.uint8)
    _load().na_gen_round_e4m3(a.ctypes.data, a.size, out.ctypes.data)
    return out


def splitmix64_at(seed: int, k: int) -> int:
    """k-th raw 64-bit output of a SplitMix64 sequence started at ``seed``."""
    return int(_load().na_gen_splitmix64_at(seed, k))


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32 (a bit shift)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def normal_f16(seed: int, shape, scale: float = 1.0, threads: int | None = None) -> np.ndarray:
    """The float32 samples of ``normal_f32`` rounded to float16 (nearest even)."""
    return normal_f32(seed, shape, scale, threads).astype(np.float16)


def qkv(seed_base: int, B: int, heads: int, grid, head_dim: int, dtype: str,
        threads: int | None = None):
    """(q, k, v) host arrays of shape [B, heads, *grid, head_dim].

    ``dtype`` is "f32" (float32 arrays), "bf16" (uint16 bit-pattern arrays),
    "f16" (float16 arrays) or "e4m3" (uint8 bit-pattern arrays).  Streams
    ``seed_base + 0/1/2`` feed q, k and v.
    """
    shape = (B, heads, *tuple(grid), head_dim)
    gens = {"f32": normal_f32, "bf16": normal_bf16_bits, "f16": normal_f16,
            "e4m3": normal_e4m3_bits}
    if dtype not in gens:
        raise ValueError(f"unknown dtype {dtype!r}")
    gen = gens[dtype]
    return tuple(gen(seed_base + t, shape, threads=threads) for t in range(3))
