"""GPU parity for float16 inputs: both kernels (the tensor-core kernel with
f16 operands and P rounded to f16, the CUDA-core kernel in fp32 arithmetic)
through the C ABI against the fp64 oracle on the same seeded float16 values.
Bar: max |out - oracle| <= 4e-3, mean <= 4e-4, |lse - oracle| <= 1e-3."""
import zlib

import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU machines skip the module
    pytest.skip("needs a CUDA device", allow_module_level=True)

import neighborhood_attention_b200 as na  # noqa: E402
from gpu_parity import assert_within, compare, host_inputs, run_gpu, sample_rows  # noqa: E402

SIMT, TC = na.NA_KERNEL_SIMT, na.NA_KERNEL_TC


def _case(grid, window, stride, d, B=1, heads=2, tile=None, mode=None):
    c = dict(B=B, heads=heads, grid=tuple(grid), window=tuple(window), stride=tuple(stride),
             tile=tile, d=d, dtype="f16")
    if mode is not None:
        c["mode"] = list(mode)
    return c


CASES = {
    "na2d_ragged": _case((37, 45), (7, 9), (1, 1), 64),
    "gna2d_strided_d128": _case((50, 44), (20, 16), (5, 4), 128),
    "sta3d_small": _case((6, 16, 40), (6, 12, 24), (2, 4, 8), 128, tile=(2, 4, 8)),
    "na1d_long": _case((1000,), (129,), (1,), 64),
    "causal1d": _case((900,), (200,), (1,), 128, mode=["causal"]),
    "batch_heads_d32": _case((20, 20), (9, 9), (3, 3), 32, B=3, heads=2),
}


@pytest.mark.parametrize("kernel", [SIMT, TC], ids=["simt", "tc"])
@pytest.mark.parametrize("name", sorted(CASES))
def test_f16_full_parity(name, kernel):
    c = CASES[name]
    if kernel == TC and c["d"] not in (64, 128):
        pytest.skip("the tensor-core kernel takes head_dim 64 or 128")
    qkv = host_inputs(c, seed=zlib.crc32(name.encode()) % 100000)
    o, l = run_gpu(c, qkv, kernel=kernel)
    assert_within(c, compare(c, qkv, o, l), f"f16 {name}/{kernel}")


def test_f16_sta3d_full_size_sampled():
    """The 3-D sliding tile workload (30x48x80, tile 6x8x8, window 18x24x40,
    24 heads, d 128) in float16, sampled rows including every corner."""
    c = _case((30, 48, 80), (18, 24, 40), (6, 8, 8), 128, heads=24, tile=(6, 8, 8))
    qkv = host_inputs(c, seed=16016)
    o, l = run_gpu(c, qkv)
    rows = sample_rows(c, 1200, seed=3)
    assert_within(c, compare(c, qkv, o, l, rows=rows), "f16 sta3d sampled")


def test_f16_and_bf16_differ_only_by_rounding():
    """The same float32 samples fed as f16 and as bf16 give outputs within the
    sum of both bars of each other (a wrong operand format would not)."""
    import numpy as np
    c16 = _case((24, 30), (7, 7), (1, 1), 64)
    cb = dict(c16, dtype="bf16")
    o16, _ = run_gpu(c16, host_inputs(c16, seed=5151), kernel=TC)
    ob, _ = run_gpu(cb, host_inputs(cb, seed=5151), kernel=TC)
    assert float(np.abs(o16 - ob).max()) < 4e-2
