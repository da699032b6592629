"""Derivation of the polynomial used by exp2_poly_x2 (na_ptx.cuh).

2^f on [-1/2, 1/2] is approximated by p(f) = 1 + c1 f + c2 f^2 + c3 f^3
(constant term fixed at 1 so that 2^0 is exact), choosing c1..c3 to minimise
the maximum relative error max |p(f) / 2^f - 1|.  That minimax problem is
linear in (c1, c2, c3, E) once sampled on a dense grid, so it is solved as a
linear program (scipy's HiGHS).  Run:

    python neighborhood_attention_b200/csrc/exp2_poly_fit.py

Expected: c1 = 0.69328292..., c2 = 0.24221096..., c3 = 0.05500892...,
maximum relative error 1.013e-4 (also with fp32 Horner evaluation).
"""
import numpy as np
from scipy.optimize import linprog


def fit(samples: int = 100001):
    xs = np.linspace(-0.5, 0.5, samples)
    w = 1.0 / 2.0 ** xs
    rows = np.stack([xs * w, xs ** 2 * w, xs ** 3 * w, -np.ones_like(xs)], 1)
    rhs = (2.0 ** xs - 1.0) * w
    a_ub = np.vstack([rows, -rows * np.array([1, 1, 1, -1])])
    b_ub = np.concatenate([rhs, -rhs])
    res = linprog([0, 0, 0, 1], A_ub=a_ub, b_ub=b_ub,
                  bounds=[(None, None)] * 3 + [(0, None)], method="highs")
    return res.x


def fp32_max_rel_err(c1, c2, c3, samples: int = 100001):
    f = np.linspace(-0.5, 0.5, samples).astype(np.float32)
    c = np.float32([c1, c2, c3])
    p = c[2]
    p = (p * f + c[1]).astype(np.float32)
    p = (p * f + c[0]).astype(np.float32)
    p = (p * f + np.float32(1.0)).astype(np.float32)
    exact = 2.0 ** f.astype(np.float64)
    return float(np.max(np.abs(p.astype(np.float64) - exact) / exact))


if __name__ == "__main__":
    c1, c2, c3, e = fit()
    print(f"c1={c1!r} c2={c2!r} c3={c3!r} minimax relative error {e:.4e}")
    print(f"fp32 Horner max relative error {fp32_max_rel_err(c1, c2, c3):.4e}")
