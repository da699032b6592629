"""GPU parity of the window-gather kernel (each query reads only its own
window's keys; for narrow windows): through the C ABI against the fp64 oracle
on identical seeded inputs, element by element over every output.  Cases
cover 1-, 2- and 3-D grids, every window mode, strides, fp32 / bf16 / f16,
head_dim 32 / 64 / 128, ragged grids whose rows straddle CTAs and heads, a
window wider than the automatic choice would give it, and full attention."""
import zlib

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU machines skip the module
    pytest.skip("needs a CUDA device", allow_module_level=True)

import neighborhood_attention_b200 as na  # noqa: E402
from gpu_parity import CONFIGS, assert_within, compare, host_inputs, run_gpu  # noqa: E402

GATHER = na.NA_KERNEL_GATHER


def _case(grid, window, stride, d, dtype="bf16", B=1, heads=2, mode=None):
    c = dict(B=B, heads=heads, grid=tuple(grid), window=tuple(window), stride=tuple(stride),
             tile=None, d=d, dtype=dtype)
    if mode is not None:
        c["mode"] = list(mode)
    return c


CASES = {
    # the 1-D causal long-sequence shape at a small size (k = 4)
    "causal1d_k4": _case((1000,), (5,), (1,), 64, B=2, heads=3, mode=["causal"]),
    "truncated1d_f16_d128": _case((777,), (9,), (1,), 128, dtype="f16", mode=["truncated"]),
    "clamped1d_strided_f32_d32": _case((300,), (17,), (4,), 32, dtype="f32", heads=3),
    "clamped2d_f32_d64": _case((23, 19), (5, 5), (1, 1), 64, dtype="f32"),
    "modes2d_strided_d32": _case((17, 31), (4, 6), (2, 3), 32, mode=["causal", "truncated"]),
    "clamped3d_d128": _case((7, 9, 11), (3, 3, 3), (1, 1, 1), 128),
    "modes3d_f16": _case((5, 12, 20), (2, 3, 5), (1, 3, 5), 64, dtype="f16", B=2, heads=1,
                         mode=["truncated", "causal", "clamped"]),
    # wider than NA_GATHER_MAX_KEYS: only by explicit choice
    "wide2d_81keys": _case((40, 40), (9, 9), (1, 1), 64),
    # the window is the whole (short) grid: full attention
    "full1d": _case((40,), (40,), (1,), 64, dtype="f16"),
    # fp32, head_dim 128: a whole warp per query
    "f32_d128": _case((50, 6), (3, 5), (1, 1), 128, dtype="f32", mode=["causal", "clamped"]),
    # a wide window whose staged tiles fit only one CTA per SM (64 queries,
    # a 320-row key box at 256 bytes a row)
    "wide1d_one_cta": _case((600,), (257,), (1,), 128, mode=["causal"]),
    # one query's key box (513 rows of K and V at 256 bytes each) exceeds the
    # shared-memory limit: the direct form, keys read from global memory
    "direct1d_wide": _case((1200,), (513,), (1,), 128, mode=["causal"]),
}


def test_wide_window_takes_the_direct_form():
    c = CASES["direct1d_wide"]
    p = na.na_plan(c["grid"], c["window"], c["stride"], None, c["d"], na.NA_BF16,
                   options=na.make_options(kernel=GATHER, window_mode=c["mode"], ndim=1))
    assert p["qblock"] == [1, 1, 1] and p["chunks_loaded"] == p["useful_pairs"]


@pytest.mark.parametrize("name", sorted(CASES))
def test_gather_full_parity(name):
    c = CASES[name]
    qkv = host_inputs(c, seed=zlib.crc32(name.encode()) % 100000)
    o, l = run_gpu(c, qkv, kernel=GATHER)
    assert_within(c, compare(c, qkv, o, l), f"{name}/gather")


def test_auto_uses_gather_and_matches_the_tile_kernels():
    """AUTO picks the gather kernel for a narrow window; the tensor-core and
    CUDA-core tile kernels meet the same bar on the same inputs, so any two of
    them differ by at most twice it (the tensor-core path also rounds P to
    bf16, which the CUDA-core kernels do not)."""
    c = _case((2048,), (5,), (1,), 64, heads=4, mode=["causal"])
    plan = na.na_plan(c["grid"], c["window"], c["stride"], None, c["d"], na.NA_BF16,
                      options=na.make_options(window_mode=c["mode"], ndim=1))
    assert plan["kernel"] == "gather"
    qkv = host_inputs(c, seed=61)
    o_auto, l_auto = run_gpu(c, qkv)
    assert_within(c, compare(c, qkv, o_auto, l_auto), "auto")
    for kernel in (na.NA_KERNEL_TC, na.NA_KERNEL_SIMT):
        o, l = run_gpu(c, qkv, kernel=kernel)
        assert_within(c, compare(c, qkv, o, l), f"kernel {kernel}")
        assert np.abs(o - o_auto).max() <= 2e-2 and np.abs(l - l_auto).max() <= 2e-3


def test_gather_deterministic():
    c = CONFIGS[6]
    qkv = host_inputs(c, seed=6006)
    o1, l1 = run_gpu(c, qkv)
    o2, l2 = run_gpu(c, qkv)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_gather_uniform_queries_give_window_sizes():
    """q = 0: every score is 0, so lse = ln(keys in the row's window) exactly
    up to fp32 rounding, and out = the window's mean of V."""
    c = _case((29, 26), (5, 3), (1, 1), 64, mode=["truncated", "causal"])
    q, k, v = host_inputs(c, seed=98)
    q = np.zeros_like(q)
    o, l = run_gpu(c, (q, k, v), kernel=GATHER)
    ref_o, ref_l = __import__("oracle").forward(q, k, v, c["grid"], c["window"], c["stride"],
                                                dtype="bf16", mode=c["mode"])
    assert np.abs(l.reshape(-1) - ref_l.reshape(-1)).max() <= 1e-5
    assert np.abs(o.reshape(ref_o.shape) - ref_o).max() <= 1e-2


def test_gather_bounded_wait_timeout_is_reported_and_recoverable():
    """The testing hook announces the first query tile's copies but issues
    none: the staged kernel's bounded waits expire, it unwinds (draining what
    was issued), na_sync_status reports NA_ERR_TIMEOUT, and the next call on
    the same context is correct."""
    from gpu_parity import to_device
    c = CASES["causal1d_k4"]
    qkv = host_inputs(c, seed=7)
    q, k, v = (to_device(a, c["dtype"]) for a in qkv)
    opts = na.make_options(kernel=GATHER, window_mode=c["mode"], ndim=1,
                           wait_timeout_ns=50_000_000, debug_flags=1)
    assert na.na_plan(c["grid"], c["window"], c["stride"], None, c["d"], na.NA_BF16,
                      options=opts)["qblock"] != [1, 1, 1]   # the staged form
    na.forward(q, k, v, c["window"], c["stride"], options=opts)
    with pytest.raises(na.NaError) as ei:
        na.na_sync_status()
    assert ei.value.status == na.NA_ERR_TIMEOUT
    na.na_sync_status()  # cleared
    o, l = run_gpu(c, qkv, kernel=GATHER)
    assert_within(c, compare(c, qkv, o, l), "after-timeout")


def _random_case(seed):
    """A seeded random problem: 1-3 dimensions, any window mode, stride and
    dilation the API accepts, every input type and head_dim."""
    rng = np.random.default_rng(seed)
    nd = int(rng.integers(1, 4))
    cap = {1: 400, 2: 40, 3: 14}[nd]
    grid = [int(rng.integers(3, cap + 1)) for _ in range(nd)]
    dil = [int(rng.integers(1, 3)) if g >= 8 else 1 for g in grid]
    window = [int(rng.integers(1, max(1, g // dl) + 1)) for g, dl in zip(grid, dil)]
    stride = [int(rng.integers(1, w + 1)) for w in window]
    mode = [["clamped", "truncated", "causal"][int(rng.integers(0, 3))] for _ in range(nd)]
    d = int(rng.choice([32, 64, 128]))
    dtype = ["bf16", "f16", "f32"][int(rng.integers(0, 3))]
    c = _case(grid, window, stride, d, dtype=dtype, heads=int(rng.integers(1, 3)), mode=mode)
    if any(x > 1 for x in dil):
        c["dil"] = tuple(dil)
    return c


@pytest.mark.parametrize("seed", range(12))
def test_gather_random_problems(seed):
    """Seeded random problems through the window-gather kernel (staged or
    direct form, one or two stages, three or five keys per step, as the plan
    picks), every output against the oracle."""
    c = _random_case(4100 + seed)
    qkv = host_inputs(c, seed=4200 + seed)
    o, l = run_gpu(c, qkv, kernel=GATHER)
    assert_within(c, compare(c, qkv, o, l), f"random {seed}: {c}")
