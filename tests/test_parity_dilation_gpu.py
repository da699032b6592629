"""GPU parity of dilated windows (per grid dimension; each residue class of
the grid is its own neighbourhood-attention problem, as the oracle's dilated
rule defines): every forward kernel through the C ABI against the fp64
oracle on identical seeded inputs, element by element over every output.
Cases: 1-, 2- and 3-D grids whose extents the dilation does not divide
(residue classes of different lengths), every window mode, strides, bf16 /
f16 / fp32 and head_dim 64 / 128."""
import zlib

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU machines skip the module
    pytest.skip("needs a CUDA device", allow_module_level=True)

import neighborhood_attention_b200 as na  # noqa: E402
from gpu_parity import assert_within, compare, host_inputs, run_gpu, sample_rows  # noqa: E402

AUTO, SIMT, TC, GATHER = (na.NA_KERNEL_AUTO, na.NA_KERNEL_SIMT, na.NA_KERNEL_TC,
                          na.NA_KERNEL_GATHER)


def _case(grid, window, stride, dil, d, dtype="bf16", B=1, heads=2, mode=None):
    c = dict(B=B, heads=heads, grid=tuple(grid), window=tuple(window), stride=tuple(stride),
             tile=None, d=d, dtype=dtype, dil=list(dil))
    if mode is not None:
        c["mode"] = list(mode)
    return c


CASES = {
    "causal1d_dil4": _case((1000,), (9,), (1,), (4,), 64, mode=["causal"]),
    "clamped2d_dil32": _case((37, 29), (5, 4), (1, 2), (3, 2), 128),
    "modes3d_dil213": _case((8, 12, 15), (3, 5, 4), (1, 1, 2), (2, 1, 3), 64, B=2, heads=1,
                            mode=["truncated", "clamped", "causal"]),
    "f16_2d_dil2": _case((30, 34), (7, 7), (1, 1), (2, 2), 64, dtype="f16", mode=["truncated"] * 2),
    # a dilated sliding-tile window: tiles of 2 x 4 x 4 inside each residue class
    "sta3d_dil": _case((6, 16, 16), (6, 8, 8), (2, 4, 4), (1, 2, 2), 128),
}
F32_CASE = _case((21, 26), (3, 5), (1, 1), (3, 2), 64, dtype="f32", mode=["causal", "clamped"])


@pytest.mark.parametrize("kernel", [AUTO, TC, SIMT, GATHER], ids=["auto", "tc", "simt", "gather"])
@pytest.mark.parametrize("name", sorted(CASES))
def test_dilated_full_parity(name, kernel):
    c = CASES[name]
    qkv = host_inputs(c, seed=zlib.crc32(name.encode()) % 100000)
    o, l = run_gpu(c, qkv, kernel=kernel)
    assert_within(c, compare(c, qkv, o, l), f"{name}/{kernel}")


@pytest.mark.parametrize("kernel", [AUTO, SIMT, GATHER], ids=["auto", "simt", "gather"])
def test_dilated_fp32_full_parity(kernel):
    qkv = host_inputs(F32_CASE, seed=515)
    o, l = run_gpu(F32_CASE, qkv, kernel=kernel)
    assert_within(F32_CASE, compare(F32_CASE, qkv, o, l), f"fp32/{kernel}")


def test_dilated_large_sampled_parity():
    """A 2-D dilated neighbourhood on a 128 x 128 grid (dilation 4, 7 x 7
    windows) through the default kernel choice, sampled rows incl. borders."""
    c = _case((128, 128), (7, 7), (1, 1), (4, 4), 64, heads=8)
    qkv = host_inputs(c, seed=4242)
    o, l = run_gpu(c, qkv)
    assert_within(c, compare(c, qkv, o, l, rows=sample_rows(c, 2000, seed=3)), "dilated 128x128")


def test_dilation_one_is_the_undilated_result():
    c = _case((40, 33), (5, 7), (1, 1), (1, 1), 64)
    qkv = host_inputs(c, seed=77)
    o1, l1 = run_gpu(c, qkv)
    c2 = dict(c)
    del c2["dil"]
    o2, l2 = run_gpu(c2, qkv)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
