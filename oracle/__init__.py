"""fp64 CPU oracle for multi-dimensional local attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never loads it and shares no code with it.

The arithmetic lives in ``na_oracle.c`` (plain C, fp64, dense mask per query);
this module compiles it with gcc and marshals numpy arrays through ctypes.
Definitions and sources are stated at the top of ``na_oracle.c``:
softmax(QK^T/sqrt(d))V restricted to the window ("pi-Attention", section 3.1
eqs. (1)-(3), section 3.2 eqs. (4)-(5)), with the window centred on the query's
stride group and clamped inside the grid ("Generalized Neighborhood Attention"
abstract; "ENA" sliding tile attention).  Per grid dimension the window may
instead be truncated at the grid border or causal ("pi-Attention" section 3.2
eq. (5)); ``mode`` arguments take "clamped" / "truncated" / "causal" (or 0 / 1
/ 2) per dimension, None meaning all clamped.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "na_oracle.c")
LIB = os.path.join(_HERE, "libna_oracle.so")
_lock = threading.Lock()
_libs: dict[str, "OracleLib"] = {}


def compile_lib(src: str, out: str) -> str:
    """Compile an oracle source file into a shared library (gcc -O2, no fast-math)."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                           "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        compile_lib(SRC, LIB)
    return LIB


class OracleLib:
    """ctypes view of one compiled oracle library (the real one, or a test mutant)."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        i32p = ctypes.POINTER(ctypes.c_int)
        lib.na_oracle_window_start.argtypes = [ctypes.c_int] * 4
        lib.na_oracle_window_start.restype = ctypes.c_int
        lib.na_oracle_window.argtypes = [ctypes.c_int] * 5 + [i32p, i32p]
        lib.na_oracle_window.restype = ctypes.c_int
        lib.na_oracle_mask_row.argtypes = [ctypes.c_int, i32p, i32p, i32p, i32p,
                                           ctypes.c_longlong, ctypes.c_void_p]
        lib.na_oracle_mask_row.restype = ctypes.c_longlong
        lib.na_oracle_mask_row_dil.argtypes = [ctypes.c_int, i32p, i32p, i32p, i32p, i32p,
                                               ctypes.c_longlong, ctypes.c_void_p]
        lib.na_oracle_mask_row_dil.restype = ctypes.c_longlong
        lib.na_oracle_dilated_window.argtypes = [ctypes.c_int] * 6 + [i32p, i32p, i32p]
        lib.na_oracle_dilated_window.restype = ctypes.c_int
        lib.na_oracle_forward_dil.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong,
            ctypes.c_int, i32p, i32p, i32p, i32p, i32p, ctypes.c_int, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_longlong, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        lib.na_oracle_forward_dil.restype = ctypes.c_int
        lib.na_oracle_forward.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong,
            ctypes.c_int, i32p, i32p, i32p, i32p, ctypes.c_int, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_longlong, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        lib.na_oracle_forward.restype = ctypes.c_int
        lib.na_oracle_block_counts.argtypes = [ctypes.c_int, i32p, i32p, i32p, i32p,
                                               ctypes.c_longlong, ctypes.c_void_p]
        lib.na_oracle_block_counts.restype = ctypes.c_int
        lib.na_oracle_backward.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
            ctypes.c_longlong, ctypes.c_int, i32p, i32p, i32p, i32p, ctypes.c_int, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        lib.na_oracle_backward.restype = ctypes.c_int
        lib.na_oracle_backward_dil.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
            ctypes.c_longlong, ctypes.c_int, i32p, i32p, i32p, i32p, i32p, ctypes.c_int,
            ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        lib.na_oracle_backward_dil.restype = ctypes.c_int
        lib.na_oracle_backward_sampled.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
            ctypes.c_longlong, ctypes.c_longlong, ctypes.c_int, i32p, i32p, i32p, i32p,
            ctypes.c_int, ctypes.c_double, ctypes.c_void_p, ctypes.c_longlong, ctypes.c_void_p,
            ctypes.c_longlong, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        lib.na_oracle_backward_sampled.restype = ctypes.c_int
        lib.na_oracle_f16_value.argtypes = [ctypes.c_uint16]
        lib.na_oracle_f16_value.restype = ctypes.c_double
        lib.na_oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.na_oracle_e4m3_value.restype = ctypes.c_double
        self.lib = lib
        self.path = path

    @staticmethod
    def _ivec(vals):
        if vals is None:
            return None
        vals = [int(x) for x in vals]
        return (ctypes.c_int * len(vals))(*vals)

    # -- window rule -------------------------------------------------------
    def window_start(self, L: int, w: int, s: int, i: int) -> int:
        r = self.lib.na_oracle_window_start(L, w, s, i)
        if r < 0:
            raise ValueError(f"invalid window arguments L={L} w={w} s={s} i={i}")
        return r

    def window(self, L: int, w: int, s: int, mode, i: int) -> tuple[int, int]:
        """The 1-D window [lo, hi) of coordinate i under ``mode``."""
        lo, hi = ctypes.c_int(), ctypes.c_int()
        r = self.lib.na_oracle_window(L, w, s, _modes([mode], 1)[0], i, ctypes.byref(lo),
                                      ctypes.byref(hi))
        if r < 0:
            raise ValueError(f"invalid window arguments L={L} w={w} s={s} mode={mode} i={i}")
        return lo.value, hi.value

    def dilated_window(self, L: int, w: int, s: int, mode, dil: int, i: int):
        """(r, lo, hi): coordinate i's keys are r + dil * t for t in [lo, hi)."""
        r, lo, hi = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
        rc = self.lib.na_oracle_dilated_window(L, w, s, _modes([mode], 1)[0], dil, i,
                                               ctypes.byref(r), ctypes.byref(lo), ctypes.byref(hi))
        if rc < 0:
            raise ValueError(f"invalid dilated window L={L} w={w} s={s} dil={dil} i={i}")
        return r.value, lo.value, hi.value

    def mask_row(self, grid, window, stride, token: int, mode=None, dilation=None) -> np.ndarray:
        grid, window, stride = _geom(grid, window, stride)
        n = int(np.prod(grid))
        out = np.zeros(n, dtype=np.uint8)
        rc = self.lib.na_oracle_mask_row_dil(len(grid), self._ivec(grid), self._ivec(window),
                                             self._ivec(stride),
                                             self._ivec(_modes(mode, len(grid))),
                                             self._ivec(_dil(dilation, len(grid))), int(token),
                                             out.ctypes.data)
        if rc < 0:
            raise ValueError("na_oracle_mask_row: invalid arguments")
        return out.astype(bool)

    # -- forward -----------------------------------------------------------
    def forward(self, q, k, v, grid, window, stride, *, dtype: str, rows=None,
                scale: float = 0.0, threads: int | None = None, mode=None, dilation=None):
        """Exact forward in fp64.

        q, k, v: arrays of shape [B, heads, *grid, d]; float32 values for
        ``dtype="f32"``, uint16 bfloat16 bit patterns for ``dtype="bf16"``,
        float16 values for ``dtype="f16"`` or uint8 OFP8 E4M3 bit patterns for
        ``dtype="e4m3"`` (the last two decoded by the C code from their bit
        patterns).
        rows: None for every query, else int64 global row ids (bh * N + token).
        Returns (out [nrows, d] float64, lse [nrows] float64); with rows=None
        out is reshaped to q's shape and lse to q's shape without d.
        """
        grid, window, stride = _geom(grid, window, stride)
        codes = {"f32": (np.float32, 0), "bf16": (np.uint16, 1), "f16": (np.float16, 2),
                 "e4m3": (np.uint8, 3)}
        if dtype not in codes:
            raise ValueError(f"unknown dtype {dtype!r}")
        want, code = codes[dtype]
        arrs = [np.ascontiguousarray(a) for a in (q, k, v)]
        for a in arrs:
            if a.dtype != want:
                raise TypeError(f"oracle expects {want} arrays for dtype={dtype}")
            if a.shape != arrs[0].shape:
                raise ValueError("q, k, v shapes differ")
        shape = arrs[0].shape
        nd = len(grid)
        if tuple(shape[2:2 + nd]) != tuple(grid) or len(shape) != nd + 3:
            raise ValueError(f"tensor shape {shape} does not match grid {grid}")
        BH = shape[0] * shape[1]
        d = shape[-1]
        N = int(np.prod(grid))
        if rows is None:
            nrows = BH * N
            rows_ptr = None
        else:
            rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
            nrows = rows.size
            rows_ptr = rows.ctypes.data
        out = np.empty((nrows, d), dtype=np.float64)
        lse = np.empty(nrows, dtype=np.float64)
        rc = self.lib.na_oracle_forward_dil(
            arrs[0].ctypes.data, arrs[1].ctypes.data, arrs[2].ctypes.data,
            code, BH, nd, self._ivec(grid), self._ivec(window),
            self._ivec(stride), self._ivec(_modes(mode, nd)), self._ivec(_dil(dilation, nd)), d,
            float(scale), rows_ptr, nrows,
            out.ctypes.data, lse.ctypes.data, int(threads or os.cpu_count() or 1))
        if rc:
            raise RuntimeError(f"na_oracle_forward failed with code {rc}")
        if rows is None:
            return out.reshape(shape).astype(np.float64), lse.reshape(shape[:-1])
        return out, lse

    def backward(self, q, k, v, dout, grid, window, stride, *, dtype: str, scale: float = 0.0,
                 threads: int | None = None, mode=None, dilation=None):
        """Exact gradients (dq, dk, dv) in fp64 for upstream gradient dout.

        q, k, v, dout: arrays of shape [B, heads, *grid, d] in the encoding of
        ``forward``'s dtype.  Returns three float64 arrays of q's shape."""
        grid, window, stride = _geom(grid, window, stride)
        codes = {"f32": (np.float32, 0), "bf16": (np.uint16, 1), "f16": (np.float16, 2),
                 "e4m3": (np.uint8, 3)}
        if dtype not in codes:
            raise ValueError(f"unknown dtype {dtype!r}")
        want, code = codes[dtype]
        arrs = [np.ascontiguousarray(a) for a in (q, k, v, dout)]
        for a in arrs:
            if a.dtype != want or a.shape != arrs[0].shape:
                raise TypeError(f"oracle expects four {want} arrays of one shape")
        shape = arrs[0].shape
        nd = len(grid)
        if tuple(shape[2:2 + nd]) != tuple(grid) or len(shape) != nd + 3:
            raise ValueError(f"tensor shape {shape} does not match grid {grid}")
        BH = shape[0] * shape[1]
        d = shape[-1]
        outs = [np.empty(shape, dtype=np.float64) for _ in range(3)]
        rc = self.lib.na_oracle_backward_dil(
            arrs[0].ctypes.data, arrs[1].ctypes.data, arrs[2].ctypes.data, arrs[3].ctypes.data,
            code, BH, nd, self._ivec(grid), self._ivec(window), self._ivec(stride),
            self._ivec(_modes(mode, nd)), self._ivec(_dil(dilation, nd)), d, float(scale),
            outs[0].ctypes.data,
            outs[1].ctypes.data, outs[2].ctypes.data, int(threads or os.cpu_count() or 1))
        if rc:
            raise RuntimeError(f"na_oracle_backward failed with code {rc}")
        return tuple(outs)

    def backward_sampled(self, q, k, v, dout, grid, window, stride, bh: int, qrows, krows, *,
                         dtype: str, scale: float = 0.0, threads: int | None = None, mode=None):
        """Exact gradients of one (batch, head) slice ``bh`` (flat index) on
        sampled rows: (dq [len(qrows), d], dk [len(krows), d], dv [len(krows), d])
        in fp64; qrows / krows are token indices within the slice."""
        grid, window, stride = _geom(grid, window, stride)
        codes = {"f32": (np.float32, 0), "bf16": (np.uint16, 1), "f16": (np.float16, 2),
                 "e4m3": (np.uint8, 3)}
        want, code = codes[dtype]
        arrs = [np.ascontiguousarray(a) for a in (q, k, v, dout)]
        for a in arrs:
            if a.dtype != want or a.shape != arrs[0].shape:
                raise TypeError(f"oracle expects four {want} arrays of one shape")
        shape = arrs[0].shape
        nd = len(grid)
        BH = shape[0] * shape[1]
        d = shape[-1]
        qr = np.ascontiguousarray(np.asarray(qrows, dtype=np.int64))
        kr = np.ascontiguousarray(np.asarray(krows, dtype=np.int64))
        dq = np.empty((qr.size, d), dtype=np.float64)
        dk = np.empty((kr.size, d), dtype=np.float64)
        dv = np.empty((kr.size, d), dtype=np.float64)
        rc = self.lib.na_oracle_backward_sampled(
            arrs[0].ctypes.data, arrs[1].ctypes.data, arrs[2].ctypes.data, arrs[3].ctypes.data,
            code, BH, int(bh), nd, self._ivec(grid), self._ivec(window), self._ivec(stride),
            self._ivec(_modes(mode, nd)), d, float(scale), qr.ctypes.data, qr.size,
            kr.ctypes.data, kr.size, dq.ctypes.data, dk.ctypes.data, dv.ctypes.data,
            int(threads or os.cpu_count() or 1))
        if rc:
            raise RuntimeError(f"na_oracle_backward_sampled failed with code {rc}")
        return dq, dk, dv

    def f16_value(self, bits: int) -> float:
        """The oracle's decoding of one binary16 bit pattern."""
        return float(self.lib.na_oracle_f16_value(int(bits)))

    def e4m3_value(self, bits: int) -> float:
        """The oracle's decoding of one OFP8 E4M3 bit pattern."""
        return float(self.lib.na_oracle_e4m3_value(int(bits)))

    # -- block counting ------------------------------------------------------
    def block_counts(self, grid, window, stride, block: int, mode=None):
        """(empty, partial, full) blk x blk tiles of the row-major attention map."""
        grid, window, stride = _geom(grid, window, stride)
        counts = np.zeros(3, dtype=np.int64)
        rc = self.lib.na_oracle_block_counts(len(grid), self._ivec(grid), self._ivec(window),
                                             self._ivec(stride), self._ivec(_modes(mode, len(grid))),
                                             int(block), counts.ctypes.data)
        if rc:
            raise ValueError("na_oracle_block_counts: invalid arguments")
        return tuple(int(c) for c in counts)


def _geom(grid, window, stride):
    grid = [int(x) for x in grid]
    window = [int(x) for x in window]
    stride = [1] * len(grid) if stride is None else [int(x) for x in stride]
    if not (len(grid) == len(window) == len(stride)):
        raise ValueError("grid, window and stride must have the same length")
    return grid, window, stride


MODES = {"clamped": 0, "truncated": 1, "causal": 2}


def _modes(mode, nd):
    """Per-dimension window modes as ints (None stays None: all clamped)."""
    if mode is None:
        return None
    if isinstance(mode, (str, int)):
        mode = [mode] * nd
    out = [MODES[m] if isinstance(m, str) else int(m) for m in mode]
    if len(out) != nd:
        raise ValueError(f"{len(out)} window modes for {nd} dimensions")
    return out


def _dil(dilation, nd):
    """Per-dimension dilation as ints (None stays None: all 1)."""
    if dilation is None:
        return None
    if isinstance(dilation, int):
        dilation = [dilation] * nd
    out = [int(x) for x in dilation]
    if len(out) != nd:
        raise ValueError(f"{len(out)} dilations for {nd} dimensions")
    return out


def load(path: str | None = None) -> OracleLib:
    """The oracle library at ``path`` (default: the real one, built on demand)."""
    with _lock:
        if path is None:
            path = build()
        if path not in _libs:
            _libs[path] = OracleLib(path)
        return _libs[path]


def window_start(L, w, s, i):
    return load().window_start(L, w, s, i)


def window(L, w, s, mode, i):
    return load().window(L, w, s, mode, i)


def mask_row(grid, window, stride, token, mode=None, dilation=None):
    return load().mask_row(grid, window, stride, token, mode, dilation)


def dilated_window(L, w, s, mode, dil, i):
    return load().dilated_window(L, w, s, mode, dil, i)


def forward(q, k, v, grid, window, stride, **kw):
    return load().forward(q, k, v, grid, window, stride, **kw)


def backward(q, k, v, dout, grid, window, stride, **kw):
    return load().backward(q, k, v, dout, grid, window, stride, **kw)


def backward_sampled(q, k, v, dout, grid, window, stride, bh, qrows, krows, **kw):
    return load().backward_sampled(q, k, v, dout, grid, window, stride, bh, qrows, krows, **kw)


def block_counts(grid, window, stride, block, mode=None):
    return load().block_counts(grid, window, stride, block, mode)
