"""GPU parity for truncated and causal windows ("pi-Attention" section 3.2
eq. (5), per grid dimension): both kernels through the C ABI against the fp64
oracle on identical seeded inputs, element by element over every output.
Cases span several query blocks and key chunks with ragged tails, windows
cut at both borders, strided (block-causal) groups, and mixed modes."""
import zlib

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU machines skip the module
    pytest.skip("needs a CUDA device", allow_module_level=True)

import neighborhood_attention_b200 as na  # noqa: E402
from gpu_parity import assert_within, compare, host_inputs, run_gpu, sample_rows  # noqa: E402

SIMT, TC = na.NA_KERNEL_SIMT, na.NA_KERNEL_TC


def _case(grid, window, stride, mode, d, dtype="bf16", B=1, heads=2, tile=None):
    return dict(B=B, heads=heads, grid=tuple(grid), window=tuple(window), stride=tuple(stride),
                tile=tile, d=d, dtype=dtype, mode=list(mode))


CASES = {
    # 1-D causal sliding window over a long sequence (k = 256 keys back)
    "causal1d_long": _case((3000,), (257,), (1,), ["causal"], 128),
    # 1-D causal, strided: block causal with 64-token groups
    "causal1d_blocks": _case((1100,), (192,), (64,), ["causal"], 64),
    # the Hilbert page's slide attention at 96x96 with an 11x11 truncated window
    "truncated2d_96": _case((96, 96), (11, 11), (1, 1), ["truncated", "truncated"], 64),
    # truncated, strided, even window, ragged grid
    "truncated2d_strided": _case((40, 37), (9, 12), (3, 4), ["truncated", "truncated"], 128),
    # video-like: causal over frames (strided), clamped in space
    "causal_t_sta3d": _case((8, 16, 24), (6, 12, 12), (2, 4, 4), ["causal", "clamped", "clamped"],
                            128, tile=(2, 4, 4)),
    # every mode at once, ragged 3-D grid
    "mixed3d": _case((9, 13, 11), (5, 6, 7), (1, 2, 1), ["truncated", "causal", "clamped"], 64,
                     B=2, heads=1),
    # causal window as long as the grid: plain causal attention
    "causal_full": _case((700,), (700,), (1,), ["causal"], 64),
}


@pytest.mark.parametrize("kernel", [SIMT, TC], ids=["simt", "tc"])
@pytest.mark.parametrize("name", sorted(CASES))
def test_mode_full_parity(name, kernel):
    c = CASES[name]
    qkv = host_inputs(c, seed=zlib.crc32(name.encode()) % 100000)
    o, l = run_gpu(c, qkv, kernel=kernel)
    assert_within(c, compare(c, qkv, o, l), f"{name}/{kernel}")


def test_mode_fp32_full_parity():
    c = _case((33, 29), (7, 5), (1, 1), ["causal", "truncated"], 32, dtype="f32", heads=3)
    qkv = host_inputs(c, seed=4242)
    o, l = run_gpu(c, qkv)
    assert_within(c, compare(c, qkv, o, l), "fp32 modes")


def test_mode_large_sampled_parity():
    """A 1-D causal workload of 32k tokens (the long-context regime of the
    pi-Attention page), sampled rows including both ends."""
    c = _case((32768,), (1025,), (1,), ["causal"], 128, B=1, heads=4)
    qkv = host_inputs(c, seed=777)
    o, l = run_gpu(c, qkv)
    rows = sample_rows(c, 1500, seed=5)
    assert_within(c, compare(c, qkv, o, l, rows=rows), "causal 32k sampled")


def test_mode_uniform_queries_give_window_sizes():
    """q = 0: lse = ln(number of keys in the row's window), which differs row
    by row near the borders for cut windows."""
    c = _case((30, 26), (9, 7), (1, 1), ["truncated", "causal"], 64)
    q, k, v = host_inputs(c, seed=99)
    q = np.zeros_like(q)
    for kernel in (SIMT, TC):
        o, l = run_gpu(c, (q, k, v), kernel=kernel)
        assert_within(c, compare(c, (q, k, v), o, l), f"uniform/{kernel}")
        counts = np.array([na.na_window_range(30, 9, 1, "truncated", i)[1] -
                           na.na_window_range(30, 9, 1, "truncated", i)[0] for i in range(30)])
        countc = np.array([j + 1 - max(0, j - 6) for j in range(26)])
        expect = np.log(np.outer(counts, countc).astype(np.float64))
        np.testing.assert_allclose(l[0, 0], expect, atol=1e-3, rtol=0)
