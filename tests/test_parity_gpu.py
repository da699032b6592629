"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
identical seeded inputs.  Small cases are compared element by element over
every output; the full-size workloads in the launch configuration the
benchmark times are compared on every element where the oracle takes
seconds, and on whole corner, edge and interior tiles of every head for the
3-D sliding tile workload."""
import zlib

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU machines skip the module
    pytest.skip("needs a CUDA device", allow_module_level=True)

import neighborhood_attention_b200 as na  # noqa: E402
from gpu_parity import (CONFIGS, assert_within, compare, host_inputs, run_gpu,  # noqa: E402
                        sample_rows, seed_for, corner_edge_interior_tiles, tile_tokens)

SIMT, TC = na.NA_KERNEL_SIMT, na.NA_KERNEL_TC


def _case(grid, window, stride, d, dtype="bf16", B=1, heads=2, tile=None):
    return dict(B=B, heads=heads, grid=tuple(grid), window=tuple(window), stride=tuple(stride),
                tile=tile, d=d, dtype=dtype)


# ---------------------------------------------------------------- small, full
SMALL = {
    "na2d_ragged": _case((37, 45), (7, 9), (1, 1), 64),
    "na2d_ragged_d128": _case((21, 19), (5, 7), (1, 1), 128, heads=3),
    "gna2d_truncated_groups": _case((50, 44), (20, 16), (5, 4), 128),
    "sta3d_small": _case((6, 16, 40), (6, 12, 24), (2, 4, 8), 64, tile=(2, 4, 8)),
    "na3d_ragged": _case((7, 9, 11), (3, 5, 7), (1, 1, 1), 128, B=2, heads=1),
    "na1d_long": _case((1000,), (129,), (1,), 64),
    "gna1d_strided": _case((777,), (96,), (32,), 128),
    "even_windows": _case((24, 30), (4, 6), (1, 2), 64),
    "full_attention": _case((24, 20), (24, 20), (1, 1), 64),
    "blocked": _case((32, 48), (8, 16), (8, 16), 64),
    "single_key": _case((16, 24), (1, 1), (1, 1), 64),
    "batch_heads": _case((20, 20), (9, 9), (3, 3), 64, B=3, heads=2),
}


@pytest.mark.parametrize("kernel", [SIMT, TC], ids=["simt", "tc"])
@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_full_parity(name, kernel):
    c = SMALL[name]
    qkv = host_inputs(c, seed=zlib.crc32(name.encode()) % 100000)
    o, l = run_gpu(c, qkv, kernel=kernel)
    assert_within(c, compare(c, qkv, o, l), f"{name}/{kernel}")


def test_fp32_config_full_parity():
    c = CONFIGS[1]
    qkv = host_inputs(c, seed_for(1))
    o, l = run_gpu(c, qkv)
    assert_within(c, compare(c, qkv, o, l), "config1")


def test_config2_full_parity_both_kernels():
    c = CONFIGS[2]
    qkv = host_inputs(c, seed_for(2))
    for kernel in (TC, SIMT):
        o, l = run_gpu(c, qkv, kernel=kernel)
        assert_within(c, compare(c, qkv, o, l), f"config2/{kernel}")


@pytest.mark.parametrize("cfg", [3, 5, 6])
def test_full_size_full_parity(cfg):
    """2-D strided (16 x 128 x 128, w 32, s 8), 3-D local (32 x 16 x 32 x 32,
    w 12 x 20 x 20) and 1-D causal (16 x 32768, w 5) workloads, in the launch
    configuration the benchmark times, compared with the oracle on every
    output element."""
    c = CONFIGS[cfg]
    qkv = host_inputs(c, seed_for(cfg))
    o, l = run_gpu(c, qkv)
    assert_within(c, compare(c, qkv, o, l), f"config{cfg}")


def test_sliding_tile_full_size_tiles_of_every_head():
    """3-D sliding tile workload (24 heads, 30 x 48 x 80, tile 6 x 8 x 8, window
    18 x 24 x 40, d 128) in the benchmark's launch configuration: every row of
    its 8 corner tiles, 4 edge tiles and 4 interior tiles, in all 24 heads
    (147,456 rows), compared with the oracle element by element."""
    c = CONFIGS[4]
    qkv = host_inputs(c, seed_for(4))
    N = int(np.prod(c["grid"]))
    corners, edges, interior = corner_edge_interior_tiles(c["grid"], c["tile"])
    toks = np.concatenate([tile_tokens(c["grid"], c["tile"], t)
                           for t in corners + edges + interior])
    BH = c["B"] * c["heads"]
    rows = (np.arange(BH, dtype=np.int64)[:, None] * N + toks[None, :]).ravel()
    o, l = run_gpu(c, qkv)
    assert_within(c, compare(c, qkv, o, l, rows=rows), "config4 tiles")


@pytest.mark.parametrize("cfg,n_rows", [(4, 1200)])
def test_full_size_sampled_parity(cfg, n_rows):
    """Uniformly drawn rows of the sliding tile workload, on top of its tiles."""
    c = CONFIGS[cfg]
    qkv = host_inputs(c, seed_for(cfg))
    rows = sample_rows(c, n_rows, seed=cfg)
    o, l = run_gpu(c, qkv)          # the launch configuration the benchmark times
    assert_within(c, compare(c, qkv, o, l, rows=rows), f"config{cfg}")


def test_tile_hint_does_not_change_results():
    c = _case((30, 32, 40), (18, 24, 40), (6, 8, 8), 128, tile=(6, 8, 8))
    qkv = host_inputs(c, seed=77)
    o1, l1 = run_gpu(c, qkv)
    o2, l2 = run_gpu(c, qkv, tile=None)
    for o, l in ((o1, l1), (o2, l2)):
        assert_within(c, compare(c, qkv, o, l, rows=sample_rows(c, 800)), "tile")


def test_uniform_queries_recover_window():
    """q = 0: every score is 0, so lse = ln(prod w) and out = mean of v over
    the window; with v = key coordinates that is start + (w-1)/2."""
    import oracle
    grid, window, stride = (20, 28), (7, 10), (1, 2)
    c = _case(grid, window, stride, 64)
    N = int(np.prod(grid))
    q = np.zeros((1, 2, *grid, 64), dtype=np.float32)
    k = np.zeros_like(q)
    v = np.zeros_like(q)
    coords = np.array(np.unravel_index(np.arange(N), grid)).T
    v.reshape(2, N, 64)[:, :, 0] = coords[:, 0]
    v.reshape(2, N, 64)[:, :, 1] = coords[:, 1]
    bits = [(a.view(np.uint32) >> 16).astype(np.uint16) for a in (q, k, v)]  # exact in bf16
    for kernel in (SIMT, TC):
        o, l = run_gpu(c, bits, kernel=kernel)
        assert np.allclose(l, np.log(np.prod(window)), atol=1e-5, rtol=0)
        for t in range(N):
            for dim in range(2):
                st = oracle.window_start(grid[dim], window[dim], stride[dim], coords[t][dim])
                exp = st + (window[dim] - 1) / 2
                got = o.reshape(2, N, 64)[:, t, dim]
                assert np.all(np.abs(got - exp) <= 2 ** -8 * max(1.0, exp)), (t, dim, got, exp)


def test_deterministic():
    c = CONFIGS[5]
    qkv = host_inputs(c, seed_for(5))
    o1, l1 = run_gpu(c, qkv)
    o2, l2 = run_gpu(c, qkv)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_bounded_wait_timeout_is_reported_and_recoverable():
    """The testing hook withholds one key chunk: the consumer's bounded wait
    expires, the kernel unwinds, na_sync_status reports NA_ERR_TIMEOUT, and
    the next call on the same context is correct."""
    from gpu_parity import to_device
    c = _case((16, 16), (5, 5), (1, 1), 64)
    qkv = host_inputs(c, seed=5)
    q, k, v = (to_device(a, "bf16") for a in qkv)
    opts = na.make_options(kernel=TC, wait_timeout_ns=50_000_000, debug_flags=1)
    na.forward(q, k, v, c["window"], c["stride"], options=opts)
    with pytest.raises(na.NaError) as ei:
        na.na_sync_status()
    assert ei.value.status == na.NA_ERR_TIMEOUT
    na.na_sync_status()  # cleared
    o, l = run_gpu(c, qkv, kernel=TC)
    assert_within(c, compare(c, qkv, o, l), "after-timeout")


def _random_tc_case(seed):
    """A seeded random problem for the tensor-core kernel: 1-3 dimensions,
    windows from a few keys to the whole grid (partial chunks on most
    blocks), any stride and window mode, bf16 or f16, head_dim 64 or 128."""
    rng = np.random.default_rng(seed)
    nd = int(rng.integers(1, 4))
    cap = {1: 1500, 2: 48, 3: 14}[nd]
    grid = [int(rng.integers(4, cap + 1)) for _ in range(nd)]
    window = [int(rng.integers(2, g + 1)) for g in grid]
    stride = [int(rng.integers(1, w + 1)) for w in window]
    mode = [["clamped", "truncated", "causal"][int(rng.integers(0, 3))] for _ in range(nd)]
    c = _case(grid, window, stride, int(rng.choice([64, 128])),
              dtype=["bf16", "f16"][int(rng.integers(0, 2))], heads=int(rng.integers(1, 3)))
    c["mode"] = mode
    return c


@pytest.mark.parametrize("seed", range(10))
def test_tc_random_problems(seed):
    """Seeded random problems through the tensor-core kernel (full and
    partial chunks, masked in tensor memory at head_dim 64 and in registers
    at 128), every output against the oracle."""
    c = _random_tc_case(5100 + seed)
    qkv = host_inputs(c, seed=5200 + seed)
    o, l = run_gpu(c, qkv, kernel=TC)
    assert_within(c, compare(c, qkv, o, l), f"random {seed}: {c}")
