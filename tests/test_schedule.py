"""The CUDA path's host-side tile scheduler against brute force: the window
rule, each query block's key box, and every chunk's empty / partial / full
label, checked pair by pair with the oracle's dense mask."""
import itertools

import numpy as np
import pytest

import neighborhood_attention_b200 as na


def test_window_rule_matches_oracle(oracle_lib):
    for L in range(1, 14):
        for w in range(1, L + 1):
            for s in range(1, w + 1):
                for i in range(L):
                    assert na.na_window_start(L, w, s, i) == oracle_lib.window_start(L, w, s, i)
    assert na.na_window_start(5, 6, 1, 0) == -1
    assert na.na_window_start(5, 3, 4, 0) == -1


def test_window_range_matches_oracle(oracle_lib):
    for L in range(1, 14):
        for w in range(1, L + 1):
            for s in range(1, w + 1):
                for i in range(L):
                    for mode in ("clamped", "truncated", "causal"):
                        assert na.na_window_range(L, w, s, mode, i) == \
                            oracle_lib.window(L, w, s, mode, i), (L, w, s, mode, i)
    assert na.na_window_range(5, 3, 1, 3, 0) is None
    assert na.na_window_range(5, 3, 1, -1, 0) is None


CASES = [
    # grid, window, stride, qblock(3-d padded), kvchunk(3-d padded)
    ([16, 16], [5, 5], [1, 1], [1, 4, 8], [1, 4, 8]),
    ([12, 20], [7, 6], [2, 3], [1, 4, 4], [1, 2, 8]),
    ([32, 32], [16, 16], [8, 8], [1, 8, 16], [1, 16, 8]),
    ([6, 8, 10], [3, 4, 5], [3, 2, 5], [2, 2, 4], [1, 4, 4]),
    ([9, 7, 5], [5, 7, 3], [1, 1, 1], [2, 4, 2], [4, 2, 2]),
    ([40], [11], [3], [1, 1, 16], [1, 1, 8]),
]
# the same with truncated / causal windows (mode per dimension)
MODE_CASES = [
    ([16, 16], [5, 5], [1, 1], [1, 4, 8], [1, 4, 8], ["truncated", "truncated"]),
    ([12, 20], [7, 6], [2, 3], [1, 4, 4], [1, 2, 8], ["causal", "truncated"]),
    ([6, 8, 10], [3, 4, 5], [3, 2, 5], [2, 2, 4], [1, 4, 4], ["causal", "clamped", "truncated"]),
    ([9, 7, 5], [5, 7, 3], [1, 1, 1], [2, 4, 2], [4, 2, 2], ["truncated", "causal", "causal"]),
    ([40], [11], [3], [1, 1, 16], [1, 1, 8], ["causal"]),
    ([64], [17], [1], [1, 1, 16], [1, 1, 16], ["causal"]),
]


@pytest.mark.parametrize("grid,window,stride,qb,kb,modes",
                         [c + (None,) for c in map(tuple, CASES)] + [tuple(c) for c in MODE_CASES])
def test_block_schedule_bruteforce(grid, window, stride, qb, kb, modes, oracle_lib):
    nd = len(grid)
    pad = 3 - nd
    g3 = [1] * pad + list(grid)
    N = int(np.prod(grid))
    nblocks = int(np.prod([-(-g3[d] // qb[d]) for d in range(3)]))
    masks = np.stack([oracle_lib.mask_row(grid, window, stride, t, mode=modes) for t in range(N)])
    mask3 = masks.reshape([N] + g3)
    for blk in range(nblocks):
        s = na.na_block_schedule(grid, window, stride, qb, kb, blk, window_mode=modes)
        o, n = s["origin"], s["extent"]
        rows = [np.ravel_multi_index(tuple(c[pad:]), grid) if nd else 0
                for c in itertools.product(*[range(o[d], o[d] + n[d]) for d in range(3)])]
        assert len(rows) == int(np.prod(n)) > 0
        m = mask3[rows]                                   # [rows, X1, X2, X3]
        keys_any = m.any(axis=0)
        keys_all = m.all(axis=0)
        # key box = bounding box of the union of the windows (which is a box)
        idx = np.nonzero(keys_any)
        for d in range(3):
            assert s["lo"][d] == idx[d].min() and s["hi"][d] == idx[d].max() + 1, (blk, d)
        box = tuple(slice(s["lo"][d], s["hi"][d]) for d in range(3))
        assert keys_any[box].all()
        # chunks of the block's own key box, row-major
        nc = [-(-(s["hi"][d] - s["lo"][d]) // kb[d]) for d in range(3)]
        assert s["nchunks"] == int(np.prod(nc))
        for c, cc in enumerate(itertools.product(*[range(x) for x in nc])):
            a = [s["lo"][d] + cc[d] * kb[d] for d in range(3)]
            inside = all(a[d] + kb[d] <= g3[d] for d in range(3))
            sl = tuple(slice(a[d], min(a[d] + kb[d], g3[d])) for d in range(3))
            sub_any, sub_all = keys_any[sl], keys_all[sl]
            if not sub_any.any():
                expect = 0
            elif inside and sub_all.all():
                expect = 2
            else:
                expect = 1
            assert s["status"][c] == expect, (blk, c, a)


def _cfg(i):
    return {
        1: dict(grid=[16, 16], window=[5, 5], stride=[1, 1], tile=None, d=32, dtype=na.NA_F32),
        2: dict(grid=[64, 64], window=[13, 13], stride=[1, 1], tile=None, d=64, dtype=na.NA_BF16),
        3: dict(grid=[128, 128], window=[32, 32], stride=[8, 8], tile=[8, 8], d=64,
                dtype=na.NA_BF16),
        4: dict(grid=[30, 48, 80], window=[18, 24, 40], stride=[6, 8, 8], tile=[6, 8, 8], d=128,
                dtype=na.NA_BF16),
        5: dict(grid=[16, 32, 32], window=[12, 20, 20], stride=[4, 4, 4], tile=[4, 4, 4], d=64,
                dtype=na.NA_BF16),
    }[i]


@pytest.mark.parametrize("i", [1, 2, 3, 4, 5])
def test_plan_statistics(i):
    c = _cfg(i)
    p = na.na_plan(c["grid"], c["window"], c["stride"], c["tile"], c["d"], c["dtype"])
    N = int(np.prod(c["grid"]))
    W = int(np.prod(c["window"]))
    assert p["useful_pairs"] == N * W
    assert p["computed_pairs"] >= p["useful_pairs"]
    if i == 1:
        # 25 keys per query: the window-gather kernel, one query per unit
        assert p["kernel"] == "gather"
        assert p["computed_pairs"] == p["useful_pairs"]
    else:
        assert p["kernel"] == "tc"
        assert np.prod(p["qblock"]) == 128 and np.prod(p["kvchunk"]) == 128
    if i == 4:
        # sliding tile attention with tile-aligned windows: every chunk is
        # full, nothing computed is masked out
        assert p["units_partial"] == 0
        assert p["computed_pairs"] == p["useful_pairs"]


@pytest.mark.parametrize("grid,window,stride,modes", [
    ([12, 10], [5, 3], [1, 1], ["truncated", "causal"]),
    ([6, 8, 9], [3, 4, 5], [3, 2, 1], ["causal", "clamped", "truncated"]),
    ([50], [17], [1], ["causal"]),
])
def test_plan_useful_pairs_with_modes(grid, window, stride, modes, oracle_lib):
    """useful_pairs = the number of (query, key) pairs the oracle's masks hold."""
    N = int(np.prod(grid))
    expect = sum(int(oracle_lib.mask_row(grid, window, stride, t, mode=modes).sum())
                 for t in range(N))
    opts = na.make_options(window_mode=modes)
    p = na.na_plan(grid, window, stride, None, 64, na.NA_BF16, options=opts)
    assert p["useful_pairs"] == expect
    assert p["computed_pairs"] >= expect


def test_speedup_bound_simulator(oracle_lib):
    """The speedup-bound simulator in na_plan: dense units over computed units.
    Perfectly block-sparse sliding tile attention reaches N / prod(w); full
    attention is 1; 1-D blocked attention with 128-token blocks agrees with
    the oracle's count of non-empty 128 x 128 tiles."""
    p = na.na_plan([30, 48, 80], [18, 24, 40], [6, 8, 8], [6, 8, 8], 128)
    assert p["units_partial"] == 0
    assert p["speedup_bound"] == pytest.approx(115200 / 17280)
    assert p["dense_pairs"] == 115200 ** 2
    p = na.na_plan([24, 40], [24, 40], [1, 1], None, 64)
    assert p["speedup_bound"] == pytest.approx(1.0)
    assert p["units_full"] + p["units_partial"] == p["dense_units"]
    p = na.na_plan([1024], [128], [128], None, 64, options=na.make_options(
        qblock=[1, 1, 128], kvchunk=[1, 1, 128]))
    e, part, full = oracle_lib.block_counts([1024], [128], [128], 128)
    assert p["dense_units"] == e + part + full == 64
    assert p["units_full"] + p["units_partial"] == part + full == 8
    assert p["speedup_bound"] == pytest.approx(8.0)


@pytest.mark.parametrize("grid,window,stride,modes,dil", [
    ([13, 10], [3, 2], [1, 2], ["clamped", "truncated"], [3, 2]),
    ([50], [5], [1], ["causal"], [4]),
    ([7, 9, 11], [2, 3, 3], [1, 1, 3], None, [2, 3, 2]),
])
@pytest.mark.parametrize("kernel", ["auto", "tc", "simt", "gather"])
def test_plan_with_dilation_counts_the_oracles_pairs(grid, window, stride, modes, dil, kernel,
                                                     oracle_lib):
    """A dilated problem is scheduled one residue class at a time; the summed
    useful pairs equal the pairs of the oracle's dilated masks."""
    sel = {"auto": na.NA_KERNEL_AUTO, "tc": na.NA_KERNEL_TC, "simt": na.NA_KERNEL_SIMT,
           "gather": na.NA_KERNEL_GATHER}[kernel]
    opts = na.make_options(kernel=sel, window_mode=modes, ndim=len(grid), dilation=dil)
    p = na.na_plan(grid, window, stride, None, 64, na.NA_BF16, options=opts)
    N = int(np.prod(grid))
    expect = sum(int(oracle_lib.mask_row(grid, window, stride, t, mode=modes, dilation=dil).sum())
                 for t in range(N))
    assert p["useful_pairs"] == expect
    assert p["computed_pairs"] >= expect
    assert p["speedup_bound"] == 0.0 and p["dense_pairs"] == N * N
