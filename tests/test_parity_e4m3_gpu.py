"""GPU parity for OFP8 E4M3 inputs: the tensor-core kernel (kind::f8f6f4
products, fp32 accumulation, bf16 out) against the fp64 oracle reading the
same E4M3 bytes.

Bar, derived from the arithmetic (the pages fix no precision for 8-bit
inputs).  q, k and v are exact on both sides, products of two E4M3 values are
exact in fp32 and the row statistics (reference maximum, row sum l, lse) stay
fp32, so lse keeps the bf16 bar, |lse - oracle| <= 1e-3.  The one new error is
P rounded to E4M3 for the second product: the kernel forms
P'_j = 2^(x_j - m_ref) >= 0 with l = sum_j P'_j >= 16 (the row's reference
lies 4 log2 units below a maximum it has seen), and rounding to nearest moves
P'_j by at most 2^-4 P'_j (half an ulp of a 3-bit mantissa) or, below the
smallest normal 2^-6, by at most 2^-10 <= 2^-14 l.  In units of the exact
softmax weights p_j = P'_j / l the error of one key is at most
u_j = max(2^-4 p_j, 2^-14); these roundings are independent and centred, so
out_ic - oracle_ic has standard deviation at most
sigma_ic = sqrt(sum_j u_j^2 v_jc^2 / 3).  The test computes sigma from the
inputs for every checked row (fp64 softmax weights over the row's window,
values decoded by torch's float8 conversion) and requires
|out - oracle| <= 7 sigma + 2^-8 |oracle| + 1e-5 element by element (7 sigma:
about 3e-12 per element for a Gaussian, and a sum of bounded uniform terms
has lighter tails; 2^-8 |oracle| covers the bf16 rounding of out) and
mean |out - oracle| <= mean sigma + 2^-8 mean |oracle|.
"""
import itertools

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU machines skip the module
    pytest.skip("needs a CUDA device", allow_module_level=True)

import neighborhood_attention_b200 as na  # noqa: E402
import oracle  # noqa: E402
import seeded_inputs  # noqa: E402
from gpu_parity import CONFIGS, sample_rows, corner_edge_interior_tiles, tile_tokens  # noqa: E402


def _decode(bits):
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def _run(c, qkv, kernel=na.NA_KERNEL_AUTO):
    q, k, v = (torch.from_numpy(a).view(torch.float8_e4m3fn).cuda() for a in qkv)
    opts = na.make_options(kernel=kernel, window_mode=c.get("mode"), ndim=len(c["grid"]),
                           dilation=c.get("dil"))
    out, lse = na.forward(q, k, v, c["window"], c["stride"], c.get("tile"), options=opts)
    na.na_sync_status()
    assert out.dtype == torch.bfloat16
    return out.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def _sigma(c, qkv, rows):
    """Per checked row and head-dim element: the standard-deviation bound of
    the E4M3 rounding of P (see the module docstring).  Rows are grouped by
    (head, window): one matrix product per group."""
    grid = c["grid"]
    N = int(np.prod(grid))
    d = c["d"]
    q, k, v = (_decode(a).reshape(-1, N, d) for a in qkv)
    scale = 1.0 / np.sqrt(d)
    coords = np.array(np.unravel_index(np.asarray(rows) % N, grid)).T
    groups = {}
    for r, row in enumerate(rows):
        bh = int(row) // N
        if c.get("dil"):     # each row on its own (small grids only)
            win = int(row)
        else:
            win = tuple(oracle.window(grid[i], c["window"][i], c["stride"][i],
                                      (c.get("mode") or ["clamped"] * len(grid))[i],
                                      int(coords[r][i]))
                        for i in range(len(grid)))
        groups.setdefault((bh, win), []).append(r)
    sig = np.empty((len(rows), d))
    for (bh, _), members in groups.items():
        t0 = int(rows[members[0]]) % N
        keys = np.flatnonzero(oracle.mask_row(grid, c["window"], c["stride"], t0, c.get("mode"),
                                              c.get("dil")))
        ts = np.asarray(rows)[members] % N
        z = (q[bh, ts] @ k[bh, keys].T) * scale
        p = np.exp(z - z.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        u2 = np.maximum(2.0 ** -4 * p, 2.0 ** -14) ** 2
        sig[members] = np.sqrt(u2 @ (v[bh, keys] ** 2) / 3.0)
    return sig


def _check(c, qkv, o, l, rows, label):
    d = c["d"]
    ref_o, ref_l = oracle.forward(*qkv, c["grid"], c["window"], c["stride"], dtype="e4m3",
                                  rows=rows, mode=c.get("mode"), dilation=c.get("dil"))
    go = o.reshape(-1, d)[rows]
    gl = l.reshape(-1)[rows]
    assert np.isfinite(go).all() and np.isfinite(gl).all(), f"{label}: non-finite output"
    sig = _sigma(c, qkv, rows)
    err = np.abs(go - ref_o)
    bound = 7.0 * sig + 2.0 ** -8 * np.abs(ref_o) + 1e-5
    worst = np.unravel_index(np.argmax(err / bound), err.shape)
    assert (err <= bound).all(), (f"{label}: |dout| {err[worst]:.3e} > bound {bound[worst]:.3e} "
                                  f"(sigma {sig[worst]:.3e}) at row {rows[worst[0]]}")
    assert err.mean() <= sig.mean() + 2.0 ** -8 * np.abs(ref_o).mean(), \
        f"{label}: mean|dout| {err.mean():.3e} > mean sigma {sig.mean():.3e}"
    dl = np.abs(gl - ref_l).max()
    assert dl <= 1e-3, f"{label}: max|dlse| {dl:.3e}"


def _case(grid, window, stride, d, B=1, heads=2, tile=None, mode=None, dil=None):
    return dict(B=B, heads=heads, grid=tuple(grid), window=tuple(window), stride=tuple(stride),
                tile=tile, d=d, dtype="e4m3", mode=mode, dil=dil)


SMALL = {
    "sta3d_d64": _case((6, 16, 40), (6, 12, 24), (2, 4, 8), 64, tile=(2, 4, 8)),
    "sta3d_d128": _case((6, 16, 40), (6, 12, 24), (2, 4, 8), 128, tile=(2, 4, 8)),
    "na2d_ragged_d128": _case((21, 19), (5, 7), (1, 1), 128, heads=3),
    "gna2d_partial_d64": _case((50, 44), (20, 16), (5, 4), 64),
    "na1d_causal_d128": _case((600,), (97,), (1,), 128, mode=["causal"]),
    "full_attention_d64": _case((24, 20), (24, 20), (1, 1), 64),
    # dilated windows (one launch per residue class, strided tensor maps)
    "dilated2d_d128": _case((23, 34), (5, 8), (1, 2), 128, dil=(3, 2),
                            mode=["clamped", "truncated"]),
}


@pytest.mark.parametrize("name", sorted(SMALL))
def test_e4m3_small_every_row(name):
    c = SMALL[name]
    qkv = seeded_inputs.qkv(7300 + len(name), c["B"], c["heads"], c["grid"], c["d"], "e4m3")
    o, l = _run(c, qkv)
    rows = np.arange(c["B"] * c["heads"] * int(np.prod(c["grid"])), dtype=np.int64)
    _check(c, qkv, o, l, rows, name)


def test_e4m3_sliding_tile_full_size_tiles():
    """3-D sliding tile workload (24 heads, 30 x 48 x 80, window 18 x 24 x 40,
    d 128) with E4M3 inputs: every row of the 8 corner, 4 edge and 4 interior
    tiles of the first and last head, plus uniformly drawn rows."""
    c = dict(CONFIGS[4], dtype="e4m3")
    qkv = seeded_inputs.qkv(7400, c["B"], c["heads"], c["grid"], c["d"], "e4m3")
    o, l = _run(c, qkv)
    N = int(np.prod(c["grid"]))
    corners, edges, interior = corner_edge_interior_tiles(c["grid"], c["tile"])
    toks = np.concatenate([tile_tokens(c["grid"], c["tile"], t)
                           for t in corners + edges + interior])
    BH = c["B"] * c["heads"]
    rows = np.unique(np.concatenate([toks, (BH - 1) * N + toks, sample_rows(c, 200, seed=74)]))
    _check(c, qkv, o, l, rows, "config4 e4m3")


def test_e4m3_local3d_full_size_sampled():
    """3-D local workload (32 heads, 16 x 32 x 32, window 12 x 20 x 20, d 64)
    with E4M3 inputs on sampled rows (grid corners and edges of the first and
    last head, uniform draws)."""
    c = dict(CONFIGS[5], dtype="e4m3")
    qkv = seeded_inputs.qkv(7500, c["B"], c["heads"], c["grid"], c["d"], "e4m3")
    o, l = _run(c, qkv)
    _check(c, qkv, o, l, sample_rows(c, 3000, seed=75), "config5 e4m3")


def test_e4m3_lazy_max_redo():
    """Planted inputs drive the reference-max redo with 8-bit operands (exact
    E4M3 values): q[..., 0] = 16 and k[..., 0] = 8 x along the outermost
    dimension (x < 8: 0 .. 56), so every later chunk beats the stale reference
    by far more than the 8-bit cap of 256 allows, and a step of 96 half way
    (row sums overflow to infinity against the stale reference)."""
    c = _case((8, 16, 32), (6, 8, 24), (2, 8, 8), 128, tile=(2, 8, 8))
    for kind in ("ramp", "step"):
        q, k, v = seeded_inputs.qkv(7600, c["B"], c["heads"], c["grid"], c["d"], "e4m3")
        x = np.arange(c["grid"][0], dtype=np.float32)
        f = 8.0 * x if kind == "ramp" else np.where(x >= c["grid"][0] // 2, 96.0, 0.0)
        fb = seeded_inputs.round_e4m3_bits(f.astype(np.float32))
        assert np.array_equal(_decode(fb), f), "planted values must be exact in E4M3"
        q = q.copy()
        k = k.copy()
        q[..., 0] = seeded_inputs.round_e4m3_bits(np.float32(16.0))
        k[..., 0] = fb.reshape(1, 1, -1, 1, 1)
        qkv = (q, k, v)
        o, l = _run(c, qkv, kernel=na.NA_KERNEL_TC)
        rows = np.arange(c["B"] * c["heads"] * int(np.prod(c["grid"])), dtype=np.int64)
        _check(c, qkv, o, l, rows, f"lazy max {kind}")


def test_e4m3_refusals():
    """E4M3 runs on the tensor-core kernel only, at head_dim 64 or 128."""
    c = SMALL["sta3d_d64"]
    q = torch.zeros((1, 1, *c["grid"], 64), dtype=torch.float8_e4m3fn, device="cuda")
    for kernel in (na.NA_KERNEL_SIMT, na.NA_KERNEL_GATHER):
        with pytest.raises(na.NaError) as e:
            na.forward(q, q, q, c["window"], c["stride"], options=na.make_options(kernel=kernel))
        assert e.value.status == na.NA_ERR_UNSUPPORTED
    q32 = torch.zeros((1, 1, 8, 8, 32), dtype=torch.float8_e4m3fn, device="cuda")
    with pytest.raises(na.NaError) as e:
        na.forward(q32, q32, q32, (3, 3))
    assert e.value.status == na.NA_ERR_UNSUPPORTED


@pytest.mark.parametrize("seed", range(6))
def test_e4m3_random_problems(seed):
    """Seeded random problems with E4M3 inputs (1-3 dimensions, any window
    mode and stride, head_dim 64 or 128), every row against the oracle."""
    rng = np.random.default_rng(7700 + seed)
    nd = int(rng.integers(1, 4))
    cap = {1: 900, 2: 40, 3: 12}[nd]
    grid = tuple(int(rng.integers(4, cap + 1)) for _ in range(nd))
    window = tuple(int(rng.integers(2, g + 1)) for g in grid)
    stride = tuple(int(rng.integers(1, w + 1)) for w in window)
    mode = [["clamped", "truncated", "causal"][int(rng.integers(0, 3))] for _ in range(nd)]
    c = _case(grid, window, stride, int(rng.choice([64, 128])), heads=int(rng.integers(1, 3)),
              mode=mode)
    qkv = seeded_inputs.qkv(7800 + seed, c["B"], c["heads"], c["grid"], c["d"], "e4m3")
    o, l = _run(c, qkv)
    rows = np.arange(c["B"] * c["heads"] * int(np.prod(c["grid"])), dtype=np.int64)
    _check(c, qkv, o, l, rows, f"random {seed}: {c}")
