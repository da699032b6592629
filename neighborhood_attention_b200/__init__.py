"""Python binding of the B200 multi-dimensional local attention library.

Argument marshalling only: every step of the forward pass runs in the CUDA
kernels of ``libna.so`` (built in-tree by ``neighborhood_attention_b200.build``).
Importing this package without the built library raises ImportError; there is
no fallback of any kind.

Functions keep the C-ABI names (``include/na.h``): ``na_forward``,
``na_forward_ex``, ``na_sync_status``, ``na_plan``, ``na_window_start``,
``na_window_range``, ``na_block_schedule``, ``na_backward``, ``na_forward_noalloc``,
``na_noalloc_status``, ``na_status_string``, ``na_last_error``.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libna.so")

NA_OK, NA_ERR_INVALID_ARG, NA_ERR_UNSUPPORTED, NA_ERR_CUDA, NA_ERR_TIMEOUT = range(5)
NA_F32, NA_BF16, NA_F16, NA_E4M3 = 0, 1, 2, 3
NA_KERNEL_AUTO, NA_KERNEL_SIMT, NA_KERNEL_TC, NA_KERNEL_GATHER = 0, 1, 2, 3
NA_GATHER_MAX_KEYS = 32
KERNEL_NAMES = {NA_KERNEL_AUTO: "auto", NA_KERNEL_SIMT: "simt", NA_KERNEL_TC: "tc",
                NA_KERNEL_GATHER: "gather"}
NA_WINDOW_CLAMPED, NA_WINDOW_TRUNCATED, NA_WINDOW_CAUSAL = range(3)
WINDOW_MODES = {"clamped": NA_WINDOW_CLAMPED, "truncated": NA_WINDOW_TRUNCATED,
                "causal": NA_WINDOW_CAUSAL}


class NaError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{_status_name(status)}: {detail}")
        self.status = status
        self.detail = detail


class na_options(ctypes.Structure):
    _fields_ = [("scale", ctypes.c_float), ("kernel", ctypes.c_int),
                ("qblock", ctypes.c_int * 3), ("kvchunk", ctypes.c_int * 3),
                ("wait_timeout_ns", ctypes.c_longlong), ("debug_flags", ctypes.c_int),
                ("window_mode", ctypes.c_int * 3), ("dilation", ctypes.c_int * 3)]


class na_plan_info(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int), ("qblock", ctypes.c_int * 3),
                ("kvchunk", ctypes.c_int * 3), ("tile", ctypes.c_int * 3),
                ("query_blocks", ctypes.c_longlong), ("ctas", ctypes.c_longlong),
                ("chunks_loaded", ctypes.c_longlong), ("units_full", ctypes.c_longlong),
                ("units_partial", ctypes.c_longlong), ("computed_pairs", ctypes.c_longlong),
                ("useful_pairs", ctypes.c_longlong), ("dense_pairs", ctypes.c_longlong),
                ("dense_units", ctypes.c_longlong), ("speedup_bound", ctypes.c_double)]

    def as_dict(self):
        out = {}
        for name, _ in self._fields_:
            v = getattr(self, name)
            out[name] = list(v) if isinstance(v, ctypes.Array) else v
        out["kernel"] = KERNEL_NAMES.get(out["kernel"], out["kernel"])
        return out


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: run `python neighborhood_attention_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    i32p = ctypes.POINTER(ctypes.c_int)
    vp = ctypes.c_void_p
    lib.na_forward.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int, ctypes.c_int, i32p, i32p, i32p,
                               i32p, i32p, ctypes.c_int, vp]
    lib.na_forward.restype = ctypes.c_int
    lib.na_forward_ex.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int, ctypes.c_int, i32p, i32p,
                                  i32p, i32p, i32p, ctypes.c_int, ctypes.POINTER(na_options), vp]
    lib.na_forward_ex.restype = ctypes.c_int
    lib.na_default_options.argtypes = []
    lib.na_default_options.restype = na_options
    lib.na_sync_status.argtypes = [vp]
    lib.na_sync_status.restype = ctypes.c_int
    lib.na_status_string.argtypes = [ctypes.c_int]
    lib.na_status_string.restype = ctypes.c_char_p
    lib.na_last_error.argtypes = []
    lib.na_last_error.restype = ctypes.c_char_p
    lib.na_plan.argtypes = [i32p, i32p, i32p, i32p, i32p, ctypes.c_int,
                            ctypes.POINTER(na_options), ctypes.POINTER(na_plan_info)]
    lib.na_plan.restype = ctypes.c_int
    lib.na_window_start.argtypes = [ctypes.c_int] * 4
    lib.na_window_start.restype = ctypes.c_int
    lib.na_window_range.argtypes = [ctypes.c_int] * 5 + [i32p, i32p]
    lib.na_window_range.restype = ctypes.c_int
    lib.na_block_schedule.argtypes = [i32p, i32p, i32p, i32p, i32p, i32p, i32p,
                                      ctypes.c_longlong, i32p, i32p, i32p, i32p, i32p, i32p, i32p,
                                      ctypes.c_int, i32p]
    lib.na_block_schedule.restype = ctypes.c_int
    lib.na_version.argtypes = []
    lib.na_version.restype = ctypes.c_int
    lib.na_forward_noalloc.argtypes = lib.na_forward_ex.argtypes
    lib.na_forward_noalloc.restype = ctypes.c_int
    lib.na_noalloc_status.argtypes = [vp]
    lib.na_noalloc_status.restype = ctypes.c_int
    lib.na_backward.argtypes = [vp] * 10 + [ctypes.c_int, ctypes.c_int, i32p, i32p, i32p, i32p,
                                            i32p, ctypes.c_int, ctypes.POINTER(na_options), vp]
    lib.na_backward.restype = ctypes.c_int
    lib.na_selftest_exp2.argtypes = [vp, vp, ctypes.c_int, vp]
    lib.na_selftest_exp2.restype = ctypes.c_int
    return lib


_lib = _load()


def _status_name(s: int) -> str:
    return _lib.na_status_string(int(s)).decode()


def _ivec(vals):
    if vals is None:
        return None
    vals = [int(x) for x in vals]
    return (ctypes.c_int * len(vals))(*vals)


def _check(status: int):
    if status != NA_OK:
        raise NaError(status, _lib.na_last_error().decode())


def na_status_string(status: int) -> str:
    return _status_name(status)


def na_last_error() -> str:
    return _lib.na_last_error().decode()


def na_version() -> int:
    return int(_lib.na_version())


def na_default_options() -> na_options:
    return _lib.na_default_options()


def window_modes(mode, ndim: int):
    """Per-dimension na_window_mode values from None (all clamped), one mode
    for every dimension, or a sequence of ndim modes ("clamped", "truncated",
    "causal" or the enum values)."""
    if mode is None:
        return [NA_WINDOW_CLAMPED] * ndim
    if isinstance(mode, (str, int)):
        mode = [mode] * ndim
    out = [WINDOW_MODES[m] if isinstance(m, str) else int(m) for m in mode]
    if len(out) != ndim:
        raise ValueError(f"{len(out)} window modes for {ndim} grid dimensions")
    return out


def make_options(kernel: int = NA_KERNEL_AUTO, scale: float = 0.0, qblock=None, kvchunk=None,
                 wait_timeout_ns: int = 0, debug_flags: int = 0, window_mode=None,
                 ndim: int | None = None, dilation=None) -> na_options:
    """na_options from keyword values; ``window_mode`` as in window_modes()
    (a single mode needs ``ndim``, or applies to all three slots);
    ``dilation``: one int per grid dimension (or one for all of them)."""
    o = na_default_options()
    if dilation is not None:
        if isinstance(dilation, int):
            dilation = [dilation] * (ndim if ndim is not None else 3)
        for i, x in enumerate(dilation):
            o.dilation[i] = int(x)
    if window_mode is not None:
        modes = window_modes(window_mode, ndim if ndim is not None else
                             (3 if isinstance(window_mode, (str, int)) else len(window_mode)))
        for i, m in enumerate(modes):
            o.window_mode[i] = m
    o.kernel = int(kernel)
    o.scale = float(scale)
    if qblock is not None:
        for i, x in enumerate(qblock):
            o.qblock[i] = int(x)
    if kvchunk is not None:
        for i, x in enumerate(kvchunk):
            o.kvchunk[i] = int(x)
    o.wait_timeout_ns = int(wait_timeout_ns)
    o.debug_flags = int(debug_flags)
    return o


def _dtype_of(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return NA_BF16
    if t.dtype == torch.float16:
        return NA_F16
    if t.dtype == torch.float32:
        return NA_F32
    if t.dtype == torch.float8_e4m3fn:
        return NA_E4M3
    raise TypeError(f"unsupported dtype {t.dtype}; use torch.bfloat16, torch.float16, "
                    "torch.float32 or torch.float8_e4m3fn")


def out_dtype(t):
    """torch dtype of `out` for inputs like `t`: the input type, except bf16
    for E4M3 inputs."""
    import torch
    return torch.bfloat16 if t.dtype == torch.float8_e4m3fn else t.dtype


def _stream_ptr(stream) -> int:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def na_forward_ex(q, k, v, out, lse, window, stride=None, tile=None, options=None, stream=None,
                  ndim=None):
    """Enqueue na_forward_ex on torch CUDA tensors.

    q, k, v, out: [B, heads, X1..Xn, d] contiguous on one CUDA device; lse:
    float32 [B, heads, X1..Xn].  ``ndim`` defaults to len(window).
    """
    nd = len(window) if ndim is None else int(ndim)
    shape = tuple(q.shape)
    if len(shape) != nd + 3:
        raise ValueError(f"q has shape {shape}; expected [B, heads, {nd} grid dims, d]")
    for name, t in (("k", k), ("v", v)):
        if tuple(t.shape) != shape or t.dtype != q.dtype:
            raise ValueError(f"{name} must match q in shape and dtype")
    if tuple(out.shape) != shape or out.dtype != out_dtype(q):
        raise ValueError(f"out must have q's shape and dtype {out_dtype(q)}")
    import torch
    if tuple(lse.shape) != shape[:-1] or lse.dtype != torch.float32:
        raise ValueError("lse must be float32 with q's shape minus head_dim")
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("lse", lse)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    dims = _ivec([nd, shape[-1]])
    st = _lib.na_forward_ex(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                            lse.data_ptr(), shape[0], shape[1], dims, _ivec(shape[2:2 + nd]),
                            _ivec(window), _ivec(stride), _ivec(tile), _dtype_of(q),
                            ctypes.byref(options) if options is not None else None,
                            _stream_ptr(stream))
    _check(st)
    return out, lse


def na_forward(q, k, v, out, lse, window, stride=None, tile=None, stream=None):
    """Enqueue na_forward (scale 1/sqrt(d), automatic kernel choice)."""
    return na_forward_ex(q, k, v, out, lse, window, stride, tile, None, stream)


def na_forward_noalloc(q, k, v, out, lse, window, stride=None, tile=None, options=None,
                       stream=None):
    """Enqueue na_forward_noalloc: the tensor-core forward pass with its device
    scratch in a fixed array inside the library, for callers that must not
    allocate device memory (see include/na.h).  Same tensor contract as
    na_forward_ex; allocates nothing (the caller passes out and lse)."""
    import torch
    nd = len(window)
    shape = tuple(q.shape)
    if len(shape) != nd + 3:
        raise ValueError(f"q has shape {shape}; expected [B, heads, {nd} grid dims, d]")
    for name, t in (("k", k), ("v", v)):
        if tuple(t.shape) != shape or t.dtype != q.dtype:
            raise ValueError(f"{name} must match q in shape and dtype")
    if tuple(out.shape) != shape or out.dtype != out_dtype(q):
        raise ValueError(f"out must have q's shape and dtype {out_dtype(q)}")
    if tuple(lse.shape) != shape[:-1] or lse.dtype != torch.float32:
        raise ValueError("lse must be float32 with q's shape minus head_dim")
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("lse", lse)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    st = _lib.na_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                 lse.data_ptr(), shape[0], shape[1], _ivec([nd, shape[-1]]),
                                 _ivec(shape[2:2 + nd]), _ivec(window), _ivec(stride),
                                 _ivec(tile), _dtype_of(q),
                                 ctypes.byref(options) if options is not None else None,
                                 _stream_ptr(stream))
    _check(st)
    return out, lse


def na_backward(q, k, v, out, dout, lse, dq, dk, dv, delta, window, stride=None, tile=None,
                options=None, stream=None):
    """Enqueue na_backward on torch CUDA tensors (see include/na.h): dq, dk, dv
    (same shape / dtype as q) and the float32 workspace delta (lse's shape)
    are written."""
    nd = len(window)
    shape = tuple(q.shape)
    if len(shape) != nd + 3:
        raise ValueError(f"q has shape {shape}; expected [B, heads, {nd} grid dims, d]")
    import torch
    for name, t in (("k", k), ("v", v), ("out", out), ("dout", dout), ("dq", dq), ("dk", dk),
                    ("dv", dv)):
        if tuple(t.shape) != shape or t.dtype != q.dtype:
            raise ValueError(f"{name} must match q in shape and dtype")
    for name, t in (("lse", lse), ("delta", delta)):
        if tuple(t.shape) != shape[:-1] or t.dtype != torch.float32:
            raise ValueError(f"{name} must be float32 with q's shape minus head_dim")
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout), ("lse", lse),
                    ("dq", dq), ("dk", dk), ("dv", dv), ("delta", delta)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    st = _lib.na_backward(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                          dout.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                          dv.data_ptr(), delta.data_ptr(), shape[0], shape[1],
                          _ivec([nd, shape[-1]]), _ivec(shape[2:2 + nd]), _ivec(window),
                          _ivec(stride), _ivec(tile), _dtype_of(q),
                          ctypes.byref(options) if options is not None else None,
                          _stream_ptr(stream))
    _check(st)
    return dq, dk, dv


def backward(q, k, v, out, lse, dout, window, stride=None, tile=None, options=None, stream=None,
             window_mode=None, dilation=None):
    """Allocate dq, dk, dv (and the delta workspace) with torch and enqueue the
    backward pass; returns (dq, dk, dv).  ``window_mode`` and ``dilation``
    as in forward() (they must match the forward's)."""
    import torch
    if window_mode is not None or dilation is not None:
        if options is None:
            options = na_default_options()
    if window_mode is not None:
        for i, m in enumerate(window_modes(window_mode, len(window))):
            options.window_mode[i] = m
    if dilation is not None:
        dl = [dilation] * len(window) if isinstance(dilation, int) else list(dilation)
        for i, x in enumerate(dl):
            options.dilation[i] = int(x)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    delta = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    return na_backward(q, k, v, out, dout, lse, dq, dk, dv, delta, window, stride, tile, options,
                       stream)


def na_selftest_exp2(x, y, stream=None):
    """y = 2^x by the kernel's FMA-pipe polynomial (float32 CUDA tensors)."""
    import torch
    if x.dtype != torch.float32 or y.dtype != torch.float32 or x.numel() != y.numel():
        raise ValueError("x and y must be float32 tensors of the same size")
    _check(_lib.na_selftest_exp2(x.data_ptr(), y.data_ptr(), x.numel(), _stream_ptr(stream)))
    return y


def na_sync_status(stream=None):
    """Synchronise the stream and raise NaError if a kernel's bounded wait expired."""
    _check(_lib.na_sync_status(_stream_ptr(stream)))


def na_noalloc_status(stream=None):
    """Synchronise the stream and raise NaError if a na_forward_noalloc kernel's
    bounded wait expired (read from the library's static array; no allocation)."""
    _check(_lib.na_noalloc_status(_stream_ptr(stream)))


def na_plan(grid, window, stride=None, tile=None, head_dim=128, dtype=NA_BF16, options=None):
    """Schedule statistics of one (batch, head) as a dict (host only, no device)."""
    info = na_plan_info()
    dims = _ivec([len(grid), head_dim])
    st = _lib.na_plan(dims, _ivec(grid), _ivec(window), _ivec(stride), _ivec(tile), int(dtype),
                      ctypes.byref(options) if options is not None else None, ctypes.byref(info))
    _check(st)
    return info.as_dict()


def na_window_start(L: int, w: int, s: int, i: int) -> int:
    return int(_lib.na_window_start(L, w, s, i))


def na_window_range(L: int, w: int, s: int, mode, i: int):
    """The kernels' 1-D window (lo, hi) of coordinate i; None on invalid input."""
    lo, hi = ctypes.c_int(), ctypes.c_int()
    m = window_modes([mode], 1)[0]
    if _lib.na_window_range(L, w, s, m, i, ctypes.byref(lo), ctypes.byref(hi)) != 0:
        return None
    return lo.value, hi.value


def na_block_schedule(grid, window, stride, qblock, kvchunk, block: int, max_chunks: int = 4096,
                      window_mode=None):
    """Key box and per-chunk status (0 empty, 1 partial, 2 full) of one query block."""
    arrs = {n: (ctypes.c_int * 3)() for n in ("origin", "extent", "lo", "hi", "ilo", "ihi")}
    status = (ctypes.c_int * max_chunks)()
    n = ctypes.c_int(0)
    dims = _ivec([len(grid), 32])
    modes = None if window_mode is None else _ivec(window_modes(window_mode, len(grid)))
    st = _lib.na_block_schedule(dims, _ivec(grid), _ivec(window), _ivec(stride), modes,
                                _ivec(qblock), _ivec(kvchunk), int(block), arrs["origin"], arrs["extent"],
                                arrs["lo"], arrs["hi"], arrs["ilo"], arrs["ihi"], status,
                                max_chunks, ctypes.byref(n))
    _check(st)
    out = {k: list(v) for k, v in arrs.items()}
    out["nchunks"] = n.value
    out["status"] = list(status[: min(n.value, max_chunks)])
    return out


def forward(q, k, v, window, stride=None, tile=None, options=None, stream=None,
            window_mode=None, dilation=None):
    """Allocate out / lse with torch and enqueue the forward pass; returns (out, lse).
    ``window_mode`` (as in window_modes()) and ``dilation`` (one int per grid
    dimension) override the corresponding options fields."""
    import torch
    if window_mode is not None or dilation is not None:
        if options is None:
            options = na_default_options()
    if window_mode is not None:
        for i, m in enumerate(window_modes(window_mode, len(window))):
            options.window_mode[i] = m
    if dilation is not None:
        dl = [dilation] * len(window) if isinstance(dilation, int) else list(dilation)
        for i, x in enumerate(dl):
            options.dilation[i] = int(x)
    out = torch.empty(q.shape, dtype=out_dtype(q), device=q.device)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    return na_forward_ex(q, k, v, out, lse, window, stride, tile, options, stream)
