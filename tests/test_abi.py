"""The C-ABI library loads on a machine without a GPU, exports every entry
point include/na.h declares, and rejects bad arguments before touching any
device."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"\b(na_[a-z_]+)\s*\(", src)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    import neighborhood_attention_b200 as na
    lib = ctypes.CDLL(na.LIB_PATH)
    names = _declared_functions()
    assert "na_forward" in names and "na_sync_status" in names
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, f"declared but not exported: {missing}"


def test_status_strings():
    import neighborhood_attention_b200 as na
    assert na.na_status_string(na.NA_OK) == "NA_OK"
    assert na.na_status_string(na.NA_ERR_TIMEOUT) == "NA_ERR_TIMEOUT"
    assert na.na_status_string(99) == "NA_ERR_UNKNOWN"
    assert na.na_version() >= 100


def _call(lib, q=16, dims=(2, 64), grid=(8, 8), window=(3, 3), stride=None, tile=None,
          dtype=1, B=1, heads=1):
    iv = lambda xs: None if xs is None else (ctypes.c_int * len(xs))(*xs)
    p = lambda x: ctypes.c_void_p(x) if x else None
    lib.na_forward.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int, ctypes.c_int] + \
        [ctypes.POINTER(ctypes.c_int)] * 5 + [ctypes.c_int, ctypes.c_void_p]
    return lib.na_forward(p(q), p(16), p(16), p(16), p(16), B, heads, iv(dims), iv(grid),
                          iv(window), iv(stride), iv(tile), dtype, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=0), 1),                                 # NULL pointer
    (dict(q=8), 1),                                 # misaligned pointer
    (dict(B=0), 1),
    (dict(dims=(4, 64)), 1),                        # ndim out of range
    (dict(dims=(2, 0)), 1),
    (dict(dims=(2, 48)), 2),                        # head_dim not supported
    (dict(grid=(0, 8)), 1),
    (dict(window=(9, 3)), 1),                       # window larger than grid
    (dict(window=(0, 3)), 1),
    (dict(stride=(4, 1)), 1),                       # stride larger than window
    (dict(stride=(0, 1)), 1),
    (dict(tile=(0, 4)), 1),
    (dict(dtype=7), 1),
    (dict(B=1 << 16, heads=1 << 15), 2),            # B * heads = 2^31 > 2^30
    (dict(dims=(3, 64), grid=(2048, 2048, 1024), window=(3, 3, 3)), 2),   # 2^32 tokens
    (dict(dims=(3, 64), grid=(2048, 1024, 1024), window=(3, 3, 3)), 2),   # exactly 2^31 tokens
])
def test_argument_errors_need_no_device(kw, expect):
    import neighborhood_attention_b200 as na
    lib = ctypes.CDLL(na.LIB_PATH)
    assert _call(lib, **kw) == expect
    lib.na_last_error.restype = ctypes.c_char_p
    assert lib.na_last_error().decode() != ""


def test_binding_refuses_cpu_tensors():
    import torch
    import neighborhood_attention_b200 as na
    q = torch.zeros(1, 1, 8, 8, 64, dtype=torch.bfloat16)
    lse = torch.zeros(1, 1, 8, 8)
    with pytest.raises(ValueError):
        na.na_forward(q, q, q, q.clone(), lse, window=(3, 3))


@pytest.mark.parametrize("bad,match", [("cpu", "CUDA tensor"), ("shape", "v must match q"),
                                       ("dtype", "dout must match q"),
                                       ("lse_dtype", "lse must be float32"),
                                       ("ndim", "expected")])
def test_backward_binding_refuses_mismatched_tensors(bad, match):
    """na.backward checks shapes, dtypes and devices before the library is
    called; CPU tensors (all this test has) are refused last."""
    import torch
    import neighborhood_attention_b200 as na
    q = torch.zeros(1, 1, 8, 8, 64, dtype=torch.bfloat16)
    t = {n: q.clone() for n in ("k", "v", "out", "dout")}
    lse = torch.zeros(1, 1, 8, 8)
    window = (3, 3)
    if bad == "shape":
        t["v"] = torch.zeros(1, 1, 8, 4, 64, dtype=torch.bfloat16)
    elif bad == "dtype":
        t["dout"] = torch.zeros(1, 1, 8, 8, 64, dtype=torch.float16)
    elif bad == "lse_dtype":
        lse = torch.zeros(1, 1, 8, 8, dtype=torch.float64)
    elif bad == "ndim":
        window = (3, 3, 3)
    with pytest.raises(ValueError, match=match):
        na.backward(q, t["k"], t["v"], t["out"], lse, t["dout"], window=window)


@pytest.mark.parametrize("mode", [3, -1, 100])
def test_bad_window_mode_is_refused(mode):
    """An unknown na_window_mode is NA_ERR_INVALID_ARG, found on the host."""
    import neighborhood_attention_b200 as na
    opts = na.make_options(window_mode=[0, mode])
    with pytest.raises(na.NaError) as e:
        na.na_plan([8, 8], [3, 3], None, None, 64, na.NA_BF16, options=opts)
    assert e.value.status == na.NA_ERR_INVALID_ARG
    assert "window_mode[1]" in e.value.detail


def test_window_mode_beyond_ndim_is_ignored():
    import neighborhood_attention_b200 as na
    opts = na.make_options(window_mode=[2, 1, 77])
    p = na.na_plan([8, 8], [3, 3], None, None, 64, na.NA_BF16, options=opts)
    assert p["useful_pairs"] > 0


@pytest.mark.parametrize("window,dtype,expect", [
    ((5, 5), "bf16", "gather"),       # 25 keys: at most NA_GATHER_MAX_KEYS
    ((4, 8), "f16", "gather"),        # 32 keys
    ((6, 6), "bf16", "tc"),           # 36 keys
    ((5, 5), "f32", "gather"),
    ((7, 7), "f32", "simt"),
])
def test_auto_sends_narrow_windows_to_the_gather_kernel(window, dtype, expect):
    import neighborhood_attention_b200 as na
    dt = {"bf16": na.NA_BF16, "f16": na.NA_F16, "f32": na.NA_F32}[dtype]
    p = na.na_plan([40, 48], list(window), None, None, 64, dt)
    assert p["kernel"] == expect
    if expect == "gather":
        # each query attends exactly its window's keys: nothing is masked; a
        # CTA stages the key box of a query tile (qblock) in shared memory
        assert p["kvchunk"] == [1, 1, 1]
        assert p["units_partial"] == 0
        assert p["units_full"] == p["useful_pairs"] == p["computed_pairs"]
        g3 = [1, 40, 48]
        assert p["ctas"] == int(np.prod([-(-g3[d] // p["qblock"][d]) for d in range(3)]))
        # every key row is staged at least once, each tile's box at most once
        assert 40 * 48 <= p["chunks_loaded"] <= p["ctas"] * np.prod(window) * 256


@pytest.mark.parametrize("grid,window,mode,d,dtype,tile", [
    # 1-D causal, k = 4, head_dim 64: 128-query tiles fill a round of the CTA's
    # 256 threads (two per query) and two stages of 50 KB leave room for two
    # CTAs per SM
    ((32768,), (5,), ["causal"], 64, "bf16", [1, 1, 128]),
    # 2-D 5 x 5: a full 128-query tile, one stage (78 KB)
    ((128, 128), (5, 5), None, 64, "bf16", [1, 8, 16]),
    # a wide window: 64-query tiles with a 320-row key box fit one CTA per SM
    ((600,), (257,), ["causal"], 128, "bf16", [1, 1, 64]),
    # one query's 513-row key box fits no shared memory: the direct form
    ((1200,), (513,), ["causal"], 128, "bf16", [1, 1, 1]),
])
def test_gather_tile_choice(grid, window, mode, d, dtype, tile):
    import neighborhood_attention_b200 as na
    dt = {"bf16": na.NA_BF16, "f16": na.NA_F16, "f32": na.NA_F32}[dtype]
    opts = na.make_options(kernel=na.NA_KERNEL_GATHER, window_mode=mode, ndim=len(grid))
    p = na.na_plan(list(grid), list(window), None, None, d, dt, options=opts)
    assert p["kernel"] == "gather" and p["qblock"] == tile


def test_gather_selector_takes_any_window_and_cut_modes():
    import neighborhood_attention_b200 as na
    opts = na.make_options(kernel=na.NA_KERNEL_GATHER, window_mode=["causal", "truncated"])
    p = na.na_plan([33, 17], [9, 7], [3, 1], None, 128, na.NA_BF16, options=opts)
    assert p["kernel"] == "gather"
    # causal over 33 with w 9, s 3; truncated over 17 with w 7: per-dimension sums
    causal = sum(min(33, (i // 3 + 1) * 3) - max(0, (i // 3 + 1) * 3 - 9) for i in range(33))
    trunc = sum(min(17, i - 3 + 7) - max(0, i - 3) for i in range(17))
    assert p["useful_pairs"] == causal * trunc == p["units_full"]


def _fake_call(lib, fn, kernel):
    import neighborhood_attention_b200 as na
    iv = lambda xs: (ctypes.c_int * len(xs))(*xs)
    o = na.make_options(kernel=kernel)
    p = ctypes.c_void_p(256)   # aligned and never dereferenced: the call fails on the host
    if fn == "na_backward":
        f = lib.na_backward
        f.argtypes = [ctypes.c_void_p] * 10 + [ctypes.c_int, ctypes.c_int] + \
            [ctypes.POINTER(ctypes.c_int)] * 5 + [ctypes.c_int, ctypes.POINTER(na.na_options),
                                                  ctypes.c_void_p]
        return f(*([p] * 10), 1, 1, iv([2, 64]), iv([8, 8]), iv([3, 3]), None, None, 1,
                 ctypes.byref(o), None)
    f = getattr(lib, fn)
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int, ctypes.c_int] + \
        [ctypes.POINTER(ctypes.c_int)] * 5 + [ctypes.c_int, ctypes.POINTER(na.na_options),
                                              ctypes.c_void_p]
    return f(*([p] * 5), 1, 1, iv([2, 64]), iv([8, 8]), iv([3, 3]), None, None, 1,
             ctypes.byref(o), None)


@pytest.mark.parametrize("fn", ["na_backward", "na_forward_noalloc"])
def test_gather_selector_is_refused_where_it_does_not_apply(fn):
    """The window-gather kernel is forward only, and the allocation-free entry
    point runs the tensor-core kernel only: both refuse the selector on the host."""
    import neighborhood_attention_b200 as na
    lib = ctypes.CDLL(na.LIB_PATH)
    assert _fake_call(lib, fn, na.NA_KERNEL_GATHER) == na.NA_ERR_UNSUPPORTED
    lib.na_last_error.restype = ctypes.c_char_p
    assert lib.na_last_error().decode() != ""


@pytest.mark.parametrize("dilation,detail", [([0, -1], "dilation[1]"), ([3, 1], "exceeds grid[0]")])
def test_bad_dilation_is_refused(dilation, detail):
    import neighborhood_attention_b200 as na
    opts = na.make_options(dilation=dilation)
    with pytest.raises(na.NaError) as e:
        na.na_plan([8, 8], [3, 3], None, None, 64, na.NA_BF16, options=opts)
    assert e.value.status == na.NA_ERR_INVALID_ARG
    assert detail in e.value.detail


def test_allocation_free_entry_refuses_dilation():
    """na_forward_noalloc runs one tensor-core launch; dilation (one launch per
    residue class) is refused on the host."""
    import neighborhood_attention_b200 as na
    lib = ctypes.CDLL(na.LIB_PATH)
    iv = lambda xs: (ctypes.c_int * len(xs))(*xs)
    o = na.make_options(dilation=[2, 2])
    p = ctypes.c_void_p(256)   # aligned and never dereferenced: the call fails on the host
    f = lib.na_forward_noalloc
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int, ctypes.c_int] + \
        [ctypes.POINTER(ctypes.c_int)] * 5 + [ctypes.c_int, ctypes.POINTER(na.na_options),
                                              ctypes.c_void_p]
    st = f(*([p] * 5), 1, 1, iv([2, 64]), iv([8, 8]), iv([3, 3]), None, None, 1, ctypes.byref(o),
           None)
    assert st == na.NA_ERR_UNSUPPORTED


_BWD_PTRS = ("q", "k", "v", "out", "dout", "lse", "dq", "dk", "dv", "delta")


def _backward_call(lib, ptr_over=None, B=1, heads=1, dims=(2, 64), grid=(8, 8), window=(3, 3),
                   stride=None, dtype=1, kernel=0):
    import neighborhood_attention_b200 as na
    iv = lambda xs: None if xs is None else (ctypes.c_int * len(xs))(*xs)
    ptrs = {n: 256 for n in _BWD_PTRS}      # aligned, never dereferenced
    ptrs.update(ptr_over or {})
    f = lib.na_backward
    f.argtypes = [ctypes.c_void_p] * 10 + [ctypes.c_int, ctypes.c_int] + \
        [ctypes.POINTER(ctypes.c_int)] * 5 + [ctypes.c_int, ctypes.POINTER(na.na_options),
                                              ctypes.c_void_p]
    o = na.make_options(kernel=kernel)
    return f(*[ctypes.c_void_p(ptrs[n]) if ptrs[n] else None for n in _BWD_PTRS], B, heads,
             iv(dims), iv(grid), iv(window), iv(stride), None, dtype, ctypes.byref(o), None)


@pytest.mark.parametrize("kw,expect", [
    *[(dict(ptr_over={n: 0}), 1) for n in _BWD_PTRS],          # each pointer NULL
    (dict(ptr_over={"q": 8}), 1),                              # 16-byte alignment
    (dict(ptr_over={"dv": 264}), 1),
    (dict(ptr_over={"lse": 258}), 1),                          # 4-byte alignment
    (dict(ptr_over={"delta": 2}), 1),
    (dict(B=0), 1),
    (dict(heads=0), 1),
    (dict(dims=(4, 64)), 1),
    (dict(dims=(2, 48)), 2),
    (dict(window=(9, 3)), 1),
    (dict(stride=(4, 1)), 1),
    (dict(dtype=0, kernel="tc"), 2),                           # tensor cores with fp32
    (dict(dtype=3), 2),                                        # no backward for E4M3
    (dict(B=1 << 16, heads=1 << 15), 2),                       # B * heads = 2^31 > 2^30
    (dict(dims=(3, 64), grid=(2048, 2048, 1024), window=(3, 3, 3)), 2),   # 2^32 tokens
    (dict(dims=(3, 64), grid=(2048, 1024, 1024), window=(3, 3, 3)), 2),   # exactly 2^31 tokens
])
def test_backward_argument_errors_need_no_device(kw, expect):
    """na_backward refuses every malformed call on the host, before any device
    work.  Fake pointers stand in for tensors, so this runs only where no
    CUDA device is visible."""
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("host refusal test with fake pointers: CPU machines only")
    import neighborhood_attention_b200 as na
    if kw.get("kernel") == "tc":
        kw = dict(kw, kernel=na.NA_KERNEL_TC)
    lib = ctypes.CDLL(na.LIB_PATH)
    assert _backward_call(lib, **kw) == expect
    lib.na_last_error.restype = ctypes.c_char_p
    assert lib.na_last_error().decode() != ""


@pytest.mark.parametrize("grid,expect", [((2048, 1024, 1024), 2),     # exactly 2^31 tokens
                                         ((2048, 2048, 1024), 2)])    # 2^32 tokens
def test_noalloc_refuses_token_counts_an_int_cannot_hold(grid, expect):
    """The allocation-free entry point shares the forward's host checks: a grid
    of 2^31 tokens or more is refused before any device work (fake pointers)."""
    import neighborhood_attention_b200 as na
    lib = ctypes.CDLL(na.LIB_PATH)
    iv = lambda xs: (ctypes.c_int * len(xs))(*xs)
    f = lib.na_forward_noalloc
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int, ctypes.c_int] + \
        [ctypes.POINTER(ctypes.c_int)] * 5 + [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    p = ctypes.c_void_p(16)
    assert f(p, p, p, p, p, 1, 1, iv((3, 64)), iv(grid), iv((3, 3, 3)), None, None, 1, None,
             None) == expect
    lib.na_last_error.restype = ctypes.c_char_p
    assert "2^31" in lib.na_last_error().decode()


def test_e4m3_plans_on_the_tensor_cores_only():
    """8-bit inputs: the tensor-core kernel is chosen even for windows the
    window-gather kernel would take; the CUDA-core kernels and head_dim 32 are
    refused on the host."""
    import neighborhood_attention_b200 as na
    plan = na.na_plan([16, 16], [3, 3], [1, 1], None, 64, na.NA_E4M3)
    assert plan["kernel"] == "tc"
    assert na.na_plan([30, 48, 80], [18, 24, 40], [6, 8, 8], [6, 8, 8], 128,
                      na.NA_E4M3)["kernel"] == "tc"
    for kernel in (na.NA_KERNEL_SIMT, na.NA_KERNEL_GATHER):
        with pytest.raises(na.NaError) as e:
            na.na_plan([16, 16], [5, 5], None, None, 64, na.NA_E4M3,
                       options=na.make_options(kernel=kernel))
        assert e.value.status == na.NA_ERR_UNSUPPORTED
    with pytest.raises(na.NaError) as e:
        na.na_plan([16, 16], [5, 5], None, None, 32, na.NA_E4M3)
    assert e.value.status == na.NA_ERR_UNSUPPORTED
    with pytest.raises(na.NaError) as e:
        na.na_plan([16, 16], [5, 5], None, None, 64, 4)
    assert e.value.status == na.NA_ERR_INVALID_ARG


def _gather_box_extent(L, w, s, mode, t):
    """Largest key-box extent along one dimension over query tiles of extent t
    (the union of the windows of the tile's first and last query), from the
    oracle's window rule."""
    import oracle
    best = 0
    for o in range(0, L, t):
        n = min(t, L - o)
        lo, _ = oracle.window(L, w, s, mode, o)
        _, hi = oracle.window(L, w, s, mode, o + n - 1)
        best = max(best, hi - lo)
    return best


def test_gather_tiles_fit_shared_memory_on_random_problems():
    """On random 1-, 2- and 3-D problems the window-gather plan's query tile is
    a box of 2^k <= 256 queries no wider than the grid needs whose staged rows
    (the tile's queries plus its largest K and V key boxes) fit one CTA's
    shared memory (220 KB with a 256-byte header); when it falls back to
    direct reads, not even a one-query tile fits."""
    import numpy as np
    import neighborhood_attention_b200 as na
    rng = np.random.default_rng(1234)
    modes = ["clamped", "truncated", "causal"]
    for _ in range(60):
        nd = int(rng.integers(1, 4))
        grid = [int(rng.integers(1, 70)) for _ in range(nd)]
        window = [int(rng.integers(1, g + 1)) for g in grid]
        stride = [int(rng.integers(1, w + 1)) for w in window]
        mode = [modes[int(rng.integers(0, 3))] for _ in range(nd)]
        d = int(rng.choice([32, 64, 128]))
        dtype, esz = [(na.NA_BF16, 2), (na.NA_F16, 2), (na.NA_F32, 4)][int(rng.integers(0, 3))]
        opts = na.make_options(kernel=na.NA_KERNEL_GATHER, window_mode=mode, ndim=nd)
        p = na.na_plan(grid, window, stride, None, d, dtype, options=opts)
        assert p["kernel"] == "gather"
        g3 = [1] * (3 - nd) + grid
        w3 = [1] * (3 - nd) + window
        s3 = [1] * (3 - nd) + stride
        m3 = ["clamped"] * (3 - nd) + mode
        t = p["qblock"]

        def footprint(tile):
            q = int(np.prod([min(tile[i], g3[i]) for i in range(3)]))
            k = int(np.prod([_gather_box_extent(g3[i], w3[i], s3[i], m3[i], tile[i])
                             for i in range(3)]))
            return 256 + (q + 2 * k) * d * esz

        # the direct form reports CTAs of several query rows each; the staged
        # form one CTA-unit per tile (a 1 x 1 x 1 tile: one per token)
        if t == [1, 1, 1] and p["ctas"] < int(np.prod(grid)):
            assert footprint([1, 1, 1]) > 220 * 1024, (grid, window, stride, mode, d)
            continue
        assert all(x >= 1 and (x & (x - 1)) == 0 for x in t) and int(np.prod(t)) <= 256
        assert all(t[i] == 1 or t[i] // 2 < g3[i] for i in range(3)), (t, g3)
        assert footprint(t) <= 220 * 1024, (grid, window, stride, mode, d, t)
