"""The FMA-pipe exponential used for part of the softmax: its coefficients
are the minimax fit (re-derived here), the algorithm meets its error bound in
float32 on the CPU, and the device code meets it on the GPU against exact
values."""
import importlib.util
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "neighborhood_attention_b200", "csrc")
BOUND = 1.02e-4


def _header_coeffs():
    src = open(os.path.join(CSRC, "na_ptx.cuh")).read()
    body = src[src.index("void exp2_poly_x2"):]
    body = body[:body.index("f2_split(p, p0, p1)")]
    vals = [float(v) for v in re.findall(r"f2\(([0-9.]+)f, \1f\)", body)]
    # c3, c2, c1, 1.0 in Horner order
    return vals


def _emulate_f32(x, c1, c2, c3):
    """The device algorithm in float32: clamp, round-to-nearest via the
    1.5 * 2^23 shifter, Horner polynomial, exponent-field add."""
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    sh = np.float32(12582912.0)
    t = (x + sh).astype(np.float32)
    j = (t - sh).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = np.float32(c3)
    p = (p * f + np.float32(c2)).astype(np.float32)
    p = (p * f + np.float32(c1)).astype(np.float32)
    p = (p * f + np.float32(1.0)).astype(np.float32)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_coefficients_are_the_minimax_fit():
    spec = importlib.util.spec_from_file_location("fit", os.path.join(CSRC, "exp2_poly_fit.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    c1, c2, c3, e = fit.fit(20001)
    vals = _header_coeffs()
    assert len(vals) == 4 and vals[3] == 1.0
    np.testing.assert_allclose(vals[:3], [c3, c2, c1], rtol=2e-5)
    assert e < BOUND


def test_float32_algorithm_meets_bound():
    c3, c2, c1, _ = _header_coeffs()
    x = np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float64)
    y = _emulate_f32(x, c1, c2, c3).astype(np.float64)
    ref = np.exp2(x.astype(np.float32).astype(np.float64))
    assert np.max(np.abs(y / ref - 1.0)) < BOUND
    ints = np.arange(-125, 9, dtype=np.float32)
    assert np.array_equal(_emulate_f32(ints, c1, c2, c3), np.exp2(ints))  # 2^j exact


@pytest.mark.gpu
def test_device_polynomial_meets_bound():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import neighborhood_attention_b200 as na
    x = torch.linspace(-125.0, 8.0, 1_000_001, dtype=torch.float32, device="cuda")
    y = torch.empty_like(x)
    na.na_selftest_exp2(x, y)
    torch.cuda.synchronize()
    ref = torch.exp2(x.double())
    rel = (y.double() / ref - 1.0).abs().max().item()
    assert rel < BOUND, rel
    ints = torch.arange(-125, 9, dtype=torch.float32, device="cuda")
    yi = torch.empty_like(ints)
    na.na_selftest_exp2(ints, yi)
    assert torch.equal(yi, torch.exp2(ints))
