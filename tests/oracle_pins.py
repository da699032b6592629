"""Pins for the fp64 oracle: checks against facts that do not come from the
oracle itself -- values the pages print, closed forms, invariants, special
cases that reduce to a dense library routine, and brute-force enumeration.

Each ``pin_*`` function takes an ``oracle.OracleLib`` and raises
``AssertionError`` on a mismatch, so the same set can be run against the real
oracle (``test_oracle_pins.py``) and against deliberately broken copies of it
(``test_oracle_mutants.py``), which must each fail at least one pin.
"""
from __future__ import annotations

import itertools
import math
import os

import numpy as np

import seeded_inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------- helpers --

def _dense_attention(q, k, v, scale):
    """Full softmax attention of one head with numpy matmuls (fp64):
    softmax(q k^T * scale) v and the row log-sum-exp."""
    s = (q @ k.T) * scale
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    return (e / l) @ v, (m + np.log(l))[:, 0]


def _randn(seed, shape):
    return seeded_inputs.normal_f32(seed, shape, threads=1)


def _leader_start(L, w, s, i):
    """Brute force: among all w-long windows that fit in [0, L), the one whose
    start is nearest to (leader - floor(w/2)), leader = member floor(s/2) of the
    stride group of i.  Exhaustive search, no clamp arithmetic."""
    g = i // s
    target = g * s + s // 2 - w // 2
    best = None
    for a in range(0, L - w + 1):
        if best is None or abs(a - target) < abs(best - target):
            best = a
    return best


def _nearest_set(L, w, i):
    """The w grid positions nearest to i (odd w, no ties possible)."""
    order = sorted(range(L), key=lambda j: (abs(j - i), j))
    return set(order[:w])


def _window_sets(grid, window, stride):
    """Per-dimension window start for every coordinate, by brute force."""
    return [[_leader_start(L, w, s, i) for i in range(L)] for L, w, s in zip(grid, window, stride)]


def _brute_mask(grid, window, stride, token):
    starts = _window_sets(grid, window, stride)
    coords = np.unravel_index(token, grid)
    N = int(np.prod(grid))
    keys = np.array(np.unravel_index(np.arange(N), grid))
    ok = np.ones(N, dtype=bool)
    for a, (L, w) in enumerate(zip(grid, window)):
        st = starts[a][coords[a]]
        ok &= (keys[a] >= st) & (keys[a] < st + w)
    return ok


# ------------------------------------------------------------------- pins --

def pin_window_bruteforce(lib):
    """Window start vs exhaustive nearest-feasible-window search, every
    (L <= 12, 1 <= w <= L, 1 <= s <= w, i)."""
    for L in range(1, 13):
        for w in range(1, L + 1):
            for s in range(1, w + 1):
                for i in range(L):
                    got = lib.window_start(L, w, s, i)
                    assert got == _leader_start(L, w, s, i), (L, w, s, i, got)


def pin_window_geometric_centre(lib):
    """When stride and window have the same parity and no clamping happens,
    the window's centre equals the centre of the query's stride group."""
    for L in range(2, 40):
        for w in range(1, L + 1):
            for s in range(1, w + 1):
                if (w - s) % 2:
                    continue
                for i in range(L):
                    g = i // s
                    start = g * s + (s - w) // 2
                    if start < 0 or start + w > L:
                        continue
                    got = lib.window_start(L, w, s, i)
                    assert 2 * got + (w - 1) == 2 * g * s + (s - 1), (L, w, s, i, got)


def pin_window_neighbourhood_metric(lib):
    """stride 1, odd w: the window is the set of the w positions nearest to i
    (neighborhood attention's clamped neighbourhood)."""
    for L in range(1, 30):
        for w in range(1, L + 1, 2):
            for i in range(L):
                st = lib.window_start(L, w, 1, i)
                assert set(range(st, st + w)) == _nearest_set(L, w, i), (L, w, i)


def pin_window_sliding_tile(lib):
    """Sliding tile attention: stride = tile t, window = n*t with n odd, t | L.
    Every query of tile g sees whole tiles g-(n-1)/2 .. g+(n-1)/2, shifted
    inside the grid at the borders."""
    for t in range(1, 9):
        for T in range(1, 9):
            L = t * T
            for n in range(1, T + 1, 2):
                w = n * t
                for i in range(L):
                    g = i // t
                    first_tile = min(max(g - (n - 1) // 2, 0), T - n)
                    assert lib.window_start(L, w, t, i) == t * first_tile, (t, T, n, i)


def pin_window_blocked(lib):
    """stride = window dividing the grid: non-overlapping blocks."""
    for w in range(1, 9):
        for nb in range(1, 7):
            L = w * nb
            for i in range(L):
                assert lib.window_start(L, w, w, i) == (i // w) * w


def pin_mask_bruteforce(lib):
    """Dense mask rows vs brute-force per-dimension membership (2D and 3D)."""
    cases = [([5, 7], [3, 4], [1, 2]), ([6, 5], [6, 2], [3, 1]), ([3, 4, 5], [2, 3, 3], [1, 3, 2]),
             ([4, 4, 6], [4, 2, 6], [2, 2, 3])]
    for grid, window, stride in cases:
        N = int(np.prod(grid))
        for t in range(N):
            got = lib.mask_row(grid, window, stride, t)
            assert np.array_equal(got, _brute_mask(grid, window, stride, t)), (grid, t)
            assert got.sum() == int(np.prod(window))


def pin_full_attention(lib):
    """window = whole grid: equals dense softmax attention (numpy matmuls)."""
    for grid, stride, d, dtype in [([7, 5], [2, 3], 16, "f32"), ([3, 4, 5], [1, 2, 5], 8, "f32"),
                                   ([23], [1], 12, "bf16"), ([6, 7], [3, 1], 16, "f16"),
                                   ([5, 9], [1, 3], 16, "e4m3")]:
        B, H = 2, 1
        shape = (B, H, *grid, d)
        if dtype == "f32":
            q, k, v = (_randn(70 + t, shape) for t in range(3))
            qf, kf, vf = q, k, v
        elif dtype == "f16":
            q, k, v = (seeded_inputs.normal_f16(85 + t, shape, threads=1) for t in range(3))
            qf, kf, vf = (a.astype(np.float64) for a in (q, k, v))
        elif dtype == "e4m3":
            q, k, v = (seeded_inputs.normal_e4m3_bits(87 + t, shape, threads=1) for t in range(3))
            qf, kf, vf = (_e4m3_reference_values(a) for a in (q, k, v))
        else:
            q, k, v = (seeded_inputs.normal_bf16_bits(80 + t, shape, threads=1) for t in range(3))
            qf, kf, vf = (seeded_inputs.bf16_bits_to_f32(a) for a in (q, k, v))
        out, lse = lib.forward(q, k, v, grid, grid, stride, dtype=dtype)
        N = int(np.prod(grid))
        for b in range(B):
            ref_o, ref_l = _dense_attention(qf[b, 0].reshape(N, d).astype(np.float64),
                                            kf[b, 0].reshape(N, d).astype(np.float64),
                                            vf[b, 0].reshape(N, d).astype(np.float64),
                                            1.0 / math.sqrt(d))
            np.testing.assert_allclose(out[b, 0].reshape(N, d), ref_o, rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[b, 0].reshape(N), ref_l, rtol=0, atol=1e-12)


def pin_blocked_attention(lib):
    """stride = window dividing the grid: each block attends densely inside
    itself (reshape into blocks, numpy dense attention per block)."""
    for grid, window, d in [([6, 8], [3, 4], 8), ([4, 6, 6], [2, 3, 2], 4)]:
        shape = (1, 2, *grid, d)
        q, k, v = (_randn(90 + t, shape) for t in range(3))
        out, lse = lib.forward(q, k, v, grid, window, window, dtype="f32")
        nd = len(grid)
        blocks = [range(L // w) for L, w in zip(grid, window)]
        for h in range(2):
            for bidx in itertools.product(*blocks):
                sl = tuple(slice(bi * w, (bi + 1) * w) for bi, w in zip(bidx, window))
                qs, ks, vs = (a[0, h][sl].reshape(-1, d).astype(np.float64) for a in (q, k, v))
                ref_o, ref_l = _dense_attention(qs, ks, vs, 1.0 / math.sqrt(d))
                np.testing.assert_allclose(out[0, h][sl].reshape(-1, d), ref_o, atol=1e-12, rtol=0)
                np.testing.assert_allclose(lse[0, h][sl].reshape(-1), ref_l, atol=1e-12, rtol=0)
        assert nd in (2, 3)


def pin_probability_rows(lib):
    """One-hot values expose the attention row itself: it sums to 1, its
    support is exactly the brute-force window, and on the support it equals a
    softmax of numpy-computed scores."""
    grid, window, stride = [4, 5], [3, 2], [1, 2]
    N = 20
    d = 32
    q = _randn(11, (1, 1, *grid, d))
    k = _randn(12, (1, 1, *grid, d))
    v = np.zeros((1, 1, *grid, d), dtype=np.float32)
    v.reshape(N, d)[np.arange(N), np.arange(N)] = 1.0
    out, lse = lib.forward(q, k, v, grid, window, stride, dtype="f32")
    P = out.reshape(N, d)[:, :N]
    qm = q.reshape(N, d).astype(np.float64)
    km = k.reshape(N, d).astype(np.float64)
    for t in range(N):
        sup = _brute_mask(grid, window, stride, t)
        assert abs(P[t].sum() - 1.0) < 1e-12
        assert np.all(P[t][~sup] == 0.0)
        assert np.all(P[t][sup] > 0.0)
        z = (km[sup] @ qm[t]) / math.sqrt(d)
        ref = np.exp(z - z.max()) / np.exp(z - z.max()).sum()
        np.testing.assert_allclose(P[t][sup], ref, atol=1e-13, rtol=0)
        np.testing.assert_allclose(lse.reshape(N)[t], z.max() + math.log(np.exp(z - z.max()).sum()),
                                   atol=1e-12, rtol=0)


def pin_uniform_queries(lib):
    """q = 0: every score is 0, so out = mean of v over the window and
    lse = ln(prod w) exactly; with v = key coordinates the output recovers the
    window start, start + (w-1)/2 per dimension."""
    for grid, window, stride in [([9, 7], [5, 4], [1, 2]), ([5, 6, 7], [3, 6, 2], [3, 2, 1])]:
        nd = len(grid)
        d = 4
        N = int(np.prod(grid))
        q = np.zeros((1, 1, *grid, d), dtype=np.float32)
        k = _randn(21, (1, 1, *grid, d))
        v = np.zeros((1, 1, *grid, d), dtype=np.float32)
        coords = np.array(np.unravel_index(np.arange(N), grid)).T
        v.reshape(N, d)[:, :nd] = coords
        v.reshape(N, d)[:, nd] = 7.0
        out, lse = lib.forward(q, k, v, grid, window, stride, dtype="f32")
        W = int(np.prod(window))
        np.testing.assert_allclose(lse.reshape(N), math.log(W), atol=1e-13, rtol=0)
        starts = _window_sets(grid, window, stride)
        for t in range(N):
            c = coords[t]
            expect = [starts[a][c[a]] + (window[a] - 1) / 2 for a in range(nd)]
            np.testing.assert_allclose(out.reshape(N, d)[t, :nd], expect, atol=1e-12, rtol=0)
            assert abs(out.reshape(N, d)[t, nd] - 7.0) < 1e-13


def pin_single_key(lib):
    """w = 1 (stride 1): each query sees only itself: out_i = v_i and
    lse_i = scale * <q_i, k_i>."""
    grid, d = [3, 4, 5], 8
    N = 60
    q, k, v = (_randn(31 + t, (1, 2, *grid, d)) for t in range(3))
    out, lse = lib.forward(q, k, v, grid, [1, 1, 1], [1, 1, 1], dtype="f32")
    np.testing.assert_allclose(out, v.astype(np.float64), atol=0, rtol=0)
    ref = (q.astype(np.float64) * k.astype(np.float64)).sum(-1) / math.sqrt(d)
    np.testing.assert_allclose(lse, ref, atol=1e-13, rtol=0)
    assert N == int(np.prod(grid))


def pin_constant_values(lib):
    """v the same vector at every key: out = that vector whatever the scores."""
    grid, d = [6, 9], 16
    q, k = (_randn(41 + t, (2, 1, *grid, d)) for t in range(2))
    row = _randn(43, (d,))
    v = np.broadcast_to(row, (2, 1, *grid, d)).copy()
    out, _ = lib.forward(q, k, v, grid, [3, 5], [1, 1], dtype="f32")
    np.testing.assert_allclose(out, np.broadcast_to(row.astype(np.float64), out.shape),
                               atol=1e-14, rtol=0)


def pin_explicit_scale(lib):
    """An explicit scale equal to 1/sqrt(d) gives the default result; scale 2x
    doubles every score, which the one-element window (w = 1) exposes in lse."""
    grid, d = [5, 5], 8
    q, k, v = (_randn(51 + t, (1, 1, *grid, d)) for t in range(3))
    o1, l1 = lib.forward(q, k, v, grid, [3, 3], [1, 1], dtype="f32")
    o2, l2 = lib.forward(q, k, v, grid, [3, 3], [1, 1], dtype="f32", scale=1 / math.sqrt(d))
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    _, l3 = lib.forward(q, k, v, grid, [1, 1], [1, 1], dtype="f32", scale=2 / math.sqrt(d))
    ref = 2 * (q.astype(np.float64) * k.astype(np.float64)).sum(-1) / math.sqrt(d)
    np.testing.assert_allclose(l3, ref, atol=1e-13, rtol=0)


def pin_row_subset(lib):
    """Computing a list of rows gives the same values as the full run."""
    grid, d = [6, 7], 8
    q, k, v = (_randn(61 + t, (2, 3, *grid, d)) for t in range(3))
    of, lf = lib.forward(q, k, v, grid, [3, 5], [1, 2], dtype="f32")
    rows = np.array([0, 5, 41, 42, 100, 251], dtype=np.int64)
    o, l = lib.forward(q, k, v, grid, [3, 5], [1, 2], dtype="f32", rows=rows)
    np.testing.assert_array_equal(o, of.reshape(-1, d)[rows])
    np.testing.assert_array_equal(l, lf.reshape(-1)[rows])


def pin_wsa_empty_blocks_golden(lib):
    """The empty-block ratios the Hilbert page prints for row-major window
    attention (Table 1, Table 2) reproduce exactly from the oracle's mask."""
    rows = _read_golden("wsa_empty_block_ratio.txt")
    for side, win, blk, pct in rows:
        e, p, f = lib.block_counts([int(side)] * 2, [int(win)] * 2, [int(win)] * 2, int(blk))
        assert round(100.0 * e / (e + p + f), 2) == round(pct, 2), (side, win, blk, e, p, f)


def pin_block_counts_closed_forms(lib):
    """Full attention has only full tiles; blocked attention whose block equals
    the tile is block-diagonal (full on the diagonal, empty elsewhere)."""
    e, p, f = lib.block_counts([8, 8], [8, 8], [1, 1], 16)
    assert (e, p, f) == (0, 0, 16)
    e, p, f = lib.block_counts([64], [16], [16], 16)
    assert (e, p, f) == (12, 0, 4)


def pin_ena_density_golden(lib):
    """ENA's example window (48x24 on a 4096-token 64x64 grid) covers about
    30% of the tokens for every query."""
    for gh, gw, wh, ww, dens, tol in _read_golden("ena_window_density.txt"):
        grid, win = [int(gh), int(gw)], [int(wh), int(ww)]
        for t in (0, 1000, 2080, 4095):
            frac = lib.mask_row(grid, win, [1, 1], t).mean()
            assert abs(frac - dens) <= tol, (t, frac)


def pin_f16_decoding(lib):
    """The oracle's binary16 decoding equals numpy's float16 -> float64
    conversion for all 65,536 bit patterns (NaN patterns decode to NaN)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([lib.f16_value(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))


def _e4m3_reference_values(bits):
    """float64 values of E4M3 bit patterns by torch's float8_e4m3fn conversion
    (a library routine, independent of the oracle's decoder)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def pin_e4m3_decoding(lib):
    """The oracle's OFP8 E4M3 decoding equals torch's float8_e4m3fn -> float64
    conversion for all 256 bit patterns (the two NaN patterns decode to NaN),
    and the format's landmarks hold: 0x7e = 448 (largest finite), 0x08 = 2^-6
    (smallest normal), 0x01 = 2^-9 (smallest subnormal), 0x38 = 1."""
    bits = np.arange(256, dtype=np.uint8)
    ref = _e4m3_reference_values(bits)
    got = np.array([lib.e4m3_value(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert nan.sum() == 2
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))
    assert lib.e4m3_value(0x7E) == 448.0 and lib.e4m3_value(0xFE) == -448.0
    assert lib.e4m3_value(0x08) == 2.0 ** -6 and lib.e4m3_value(0x01) == 2.0 ** -9
    assert lib.e4m3_value(0x38) == 1.0 and lib.e4m3_value(0x00) == 0.0


# ------------------------------------------------- truncated / causal modes --

def _eq5_set(L, k, i, causal):
    """"pi-Attention" section 3.2 eq. (5) written out: the causal
    neighbourhood {j : max(0, i-k) <= j <= i} or the bidirectional one
    {j : |j - i| <= k}, restricted to the grid [0, L)."""
    if causal:
        return {j for j in range(L) if max(0, i - k) <= j <= i}
    return {j for j in range(L) if abs(j - i) <= k}


def _mode_set(L, w, s, mode, i):
    """Brute-force 1-D window of coordinate i for every mode.
    clamped:   the brute-force nearest feasible window (_leader_start).
    truncated: the clamped window of the same query on a grid padded by a
               multiple of s on both sides (wide enough that nothing is
               clamped there), mapped back and cut to [0, L).
    causal:    the w positions ending with the largest coordinate of i's
               stride group, cut to [0, L)."""
    if mode == "clamped":
        st = _leader_start(L, w, s, i)
        return set(range(st, st + w))
    if mode == "truncated":
        P = s * (w + 1)
        st = _leader_start(L + 2 * P, w, s, i + P) - P
        return {j for j in range(st, st + w) if 0 <= j < L}
    last = max(m for m in range(i, i + s) if m // s == i // s)
    return {j for j in range(L) if 0 <= last - j < w}


def _mode_mask(grid, window, stride, modes, token):
    coords = np.unravel_index(token, grid)
    N = int(np.prod(grid))
    keys = np.array(np.unravel_index(np.arange(N), grid))
    ok = np.ones(N, dtype=bool)
    for a, (L, w, s, m) in enumerate(zip(grid, window, stride, modes)):
        ok &= np.isin(keys[a], sorted(_mode_set(L, w, s, m, int(coords[a]))))
    return ok


def pin_truncated_eq5(lib):
    """stride 1, w = 2k + 1: the truncated window is eq. (5)'s bidirectional
    neighbourhood |j - i| <= k cut to the grid."""
    for L in range(1, 24):
        for w in range(1, L + 1, 2):
            for i in range(L):
                lo, hi = lib.window(L, w, 1, "truncated", i)
                assert set(range(lo, hi)) == _eq5_set(L, (w - 1) // 2, i, False), (L, w, i)


def pin_causal_eq5(lib):
    """stride 1, w = k + 1: the causal window is eq. (5)'s causal
    neighbourhood max(0, i-k) <= j <= i (self included)."""
    for L in range(1, 24):
        for w in range(1, L + 1):
            for i in range(L):
                lo, hi = lib.window(L, w, 1, "causal", i)
                assert set(range(lo, hi)) == _eq5_set(L, w - 1, i, True), (L, w, i)


def pin_modes_strided(lib):
    """Every mode, stride and window on short grids vs the brute-force sets:
    truncated = the unclamped centred window cut to the grid, causal = the w
    positions ending with the query's stride group."""
    for L in range(1, 15):
        for w in range(1, L + 1):
            for s in range(1, w + 1):
                for i in range(L):
                    for mode in ("clamped", "truncated", "causal"):
                        lo, hi = lib.window(L, w, s, mode, i)
                        assert set(range(lo, hi)) == _mode_set(L, w, s, mode, i), \
                            (L, w, s, mode, i)


def pin_mode_mask_bruteforce(lib):
    """Dense mask rows with a different mode per dimension vs the product of
    the brute-force 1-D sets."""
    cases = [([7, 6], [5, 3], [1, 1], ["truncated", "causal"]),
             ([6, 8], [4, 5], [2, 1], ["causal", "clamped"]),
             ([4, 5, 6], [3, 3, 4], [1, 3, 2], ["causal", "truncated", "truncated"]),
             ([9], [4], [2], ["causal"])]
    for grid, window, stride, modes in cases:
        N = int(np.prod(grid))
        for t in range(N):
            got = lib.mask_row(grid, window, stride, t, mode=modes)
            assert np.array_equal(got, _mode_mask(grid, window, stride, modes, t)), (grid, t)


def pin_causal_full_sdpa(lib):
    """A causal window as long as the grid is causal attention: equals
    torch's scaled_dot_product_attention(is_causal=True) in fp64.  Causal in
    the outer dimension only, with whole-grid windows elsewhere, is
    frame-causal attention: SDPA with a block lower-triangular boolean mask."""
    import torch
    import torch.nn.functional as F
    d = 16
    L = 37
    q, k, v = (_randn(100 + t, (2, 3, L, d)) for t in range(3))
    out, lse = lib.forward(q, k, v, [L], [L], [1], dtype="f32", mode=["causal"])
    qt, kt, vt = (torch.from_numpy(a.astype(np.float64)) for a in (q, k, v))
    ref = F.scaled_dot_product_attention(qt, kt, vt, is_causal=True).numpy()
    np.testing.assert_allclose(out, ref, atol=1e-12, rtol=0)
    s = (qt @ kt.transpose(-1, -2)) / math.sqrt(d)
    s = s.masked_fill(~torch.ones(L, L, dtype=torch.bool).tril(), -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), atol=1e-12, rtol=0)

    grid = [5, 3, 4]
    N = 60
    q, k, v = (_randn(110 + t, (1, 2, *grid, d)) for t in range(3))
    out, _ = lib.forward(q, k, v, grid, grid, [1, 1, 1], dtype="f32",
                         mode=["causal", "clamped", "clamped"])
    frame = torch.arange(N) // 12
    mask = frame[None, :] <= frame[:, None]
    qt, kt, vt = (torch.from_numpy(a.reshape(1, 2, N, d).astype(np.float64)) for a in (q, k, v))
    ref = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask).numpy()
    np.testing.assert_allclose(out.reshape(1, 2, N, d), ref, atol=1e-12, rtol=0)


def pin_mode_uniform_queries(lib):
    """q = 0 with cut windows: every row averages v over its own (smaller)
    window, so lse = ln(window size) and the mean key coordinate is the centre
    of the brute-force set, per row."""
    for grid, window, stride, modes in [([9, 8], [5, 4], [1, 2], ["truncated", "causal"]),
                                        ([6, 5, 7], [3, 5, 3], [3, 1, 1],
                                         ["causal", "clamped", "truncated"])]:
        nd = len(grid)
        d = 4
        N = int(np.prod(grid))
        q = np.zeros((1, 1, *grid, d), dtype=np.float32)
        k = _randn(121, (1, 1, *grid, d))
        v = np.zeros((1, 1, *grid, d), dtype=np.float32)
        coords = np.array(np.unravel_index(np.arange(N), grid)).T
        v.reshape(N, d)[:, :nd] = coords
        out, lse = lib.forward(q, k, v, grid, window, stride, dtype="f32", mode=modes)
        for t in range(N):
            sets = [_mode_set(grid[a], window[a], stride[a], modes[a], int(coords[t][a]))
                    for a in range(nd)]
            count = int(np.prod([len(x) for x in sets]))
            assert abs(lse.reshape(N)[t] - math.log(count)) < 1e-13, (t, count)
            expect = [np.mean(sorted(x)) for x in sets]
            np.testing.assert_allclose(out.reshape(N, d)[t, :nd], expect, atol=1e-12, rtol=0)


# ------------------------------------------------------------- dilation --
# Dilation is not defined by the pages (only named as a related pattern); the
# reading: the window rule applied inside each residue class modulo dil.  The
# brute force below builds each residue class's coordinate list explicitly
# and indexes into it, so it shares no arithmetic with the oracle's
# length / position formulas.

def _dilated_set(L, w, s, mode, dil, i):
    sub = [c for c in range(L) if c % dil == i % dil]      # the residue class, in order
    p = sub.index(i)
    return {sub[t] for t in _mode_set(len(sub), w, s, mode, p)}


def pin_dilated_window_bruteforce(lib):
    """Every mode, stride, dilation and window with w * dil <= L on short
    grids (ragged residue classes included) vs the explicit residue lists."""
    for L in range(1, 15):
        for dil in range(1, L + 1):
            for w in range(1, L // dil + 1):
                for s in range(1, w + 1):
                    for i in range(L):
                        for mode in ("clamped", "truncated", "causal"):
                            r, lo, hi = lib.dilated_window(L, w, s, mode, dil, i)
                            got = {r + dil * t for t in range(lo, hi)}
                            assert got == _dilated_set(L, w, s, mode, dil, i), \
                                (L, w, s, mode, dil, i)


def pin_dilated_mask_bruteforce(lib):
    """Dense mask rows with dilation (and modes) per dimension vs the
    product of the brute-force 1-D sets."""
    cases = [([11, 7], [3, 2], [1, 1], ["clamped", "causal"], [3, 2]),
             ([9, 10], [2, 3], [2, 1], ["truncated", "clamped"], [4, 3]),
             ([5, 6, 7], [2, 3, 3], [1, 3, 1], ["causal", "truncated", "clamped"], [2, 2, 2])]
    for grid, window, stride, modes, dil in cases:
        N = int(np.prod(grid))
        keys = np.array(np.unravel_index(np.arange(N), grid))
        for t in range(N):
            coords = np.unravel_index(t, grid)
            ok = np.ones(N, dtype=bool)
            for a in range(len(grid)):
                ok &= np.isin(keys[a], sorted(_dilated_set(grid[a], window[a], stride[a], modes[a],
                                                           dil[a], int(coords[a]))))
            got = lib.mask_row(grid, window, stride, t, mode=modes, dilation=dil)
            assert np.array_equal(got, ok), (grid, dil, t)


def pin_dilated_residue_subgrids(lib):
    """Dilated attention is undilated attention on each residue-class
    sub-grid: slice q, k, v with step dil, run the (undilated, separately
    pinned) forward on the slice, compare with the dilated forward's rows for
    those queries.  Grids whose extents dil does not divide give sub-grids of
    different lengths."""
    d = 8
    for grid, window, stride, modes, dil in [([13, 10], [3, 2], [1, 2], ["clamped", "truncated"],
                                              [3, 2]),
                                             ([7, 9], [2, 3], [1, 1], ["causal", "causal"], [2, 3])]:
        q, k, v = (_randn(300 + t, (1, 2, *grid, d)) for t in range(3))
        out, lse = lib.forward(q, k, v, grid, window, stride, dtype="f32", mode=modes,
                               dilation=dil)
        for r0 in range(dil[0]):
            for r1 in range(dil[1]):
                sl = (slice(None), slice(None), slice(r0, None, dil[0]), slice(r1, None, dil[1]))
                qs, ks, vs = (np.ascontiguousarray(a[sl]) for a in (q, k, v))
                sub = list(qs.shape[2:4])
                o2, l2 = lib.forward(qs, ks, vs, sub, window, stride, dtype="f32", mode=modes)
                np.testing.assert_allclose(out[sl], o2, atol=1e-13, rtol=0)
                np.testing.assert_allclose(lse[sl[:4]], l2, atol=1e-13, rtol=0)


def pin_dilated_backward_subgrids(lib):
    """The gradients of dilated attention are those of undilated attention on
    each residue-class sub-grid (the sub-grids do not interact)."""
    d = 6
    grid, window, stride, modes, dil = [11, 9], [3, 2], [1, 1], ["truncated", "causal"], [2, 3]
    q, k, v, do = (_randn(330 + t, (1, 2, *grid, d)) for t in range(4))
    dq, dk, dv = lib.backward(q, k, v, do, grid, window, stride, dtype="f32", mode=modes,
                              dilation=dil)
    for r0 in range(dil[0]):
        for r1 in range(dil[1]):
            sl = (slice(None), slice(None), slice(r0, None, dil[0]), slice(r1, None, dil[1]))
            qs, ks, vs, ds = (np.ascontiguousarray(a[sl]) for a in (q, k, v, do))
            g2 = lib.backward(qs, ks, vs, ds, list(qs.shape[2:4]), window, stride, dtype="f32",
                              mode=modes)
            for a, b in zip((dq, dk, dv), g2):
                np.testing.assert_allclose(a[sl], b, atol=1e-12, rtol=0)


def pin_sa_empty_blocks_golden(lib):
    """The Hilbert page's empty-block ratio for row-major slide attention
    (Table 3, SA (Flex) at 96x96) reproduces from the truncated window."""
    for side, win, blk, pct in _read_golden("sa_empty_block_ratio.txt"):
        e, p, f = lib.block_counts([int(side)] * 2, [int(win)] * 2, [1, 1], int(blk),
                                   mode="truncated")
        assert round(100.0 * e / (e + p + f), 2) == round(pct, 2), (side, win, blk, e, p, f)


# --------------------------------------------------------------- backward --

def pin_backward_finite_differences(lib):
    """Gradients of L = sum(out * dO) against central differences of the
    oracle's own (pinned) forward: every element of dq, dk and dv on a small
    2-D problem with mixed window modes and a stride.  The perturbation is
    measured on the float32 values actually fed in."""
    grid, window, stride, modes = [4, 5], [3, 3], [1, 2], ["clamped", "causal"]
    d = 3
    shape = (1, 1, *grid, d)
    q, k, v, do = (_randn(150 + t, shape).astype(np.float64).astype(np.float32) for t in range(4))
    dq, dk, dv = lib.backward(q, k, v, do, grid, window, stride, dtype="f32", mode=modes)

    def loss(qq, kk, vv):
        out, _ = lib.forward(qq, kk, vv, grid, window, stride, dtype="f32", mode=modes)
        return float((out * do.astype(np.float64)).sum())

    h = 1e-2
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        for idx in np.ndindex(*shape):
            args = [q.copy(), k.copy(), v.copy()]
            x0 = args[which][idx]
            args[which][idx] = np.float32(x0 + h)
            up = args[which][idx]
            fp = loss(*args)
            args[which][idx] = np.float32(x0 - h)
            dn = args[which][idx]
            fm = loss(*args)
            num = (fp - fm) / (float(up) - float(dn))
            assert abs(num - grad[idx]) <= 2e-4 * max(1.0, abs(num)), (which, idx, num, grad[idx])


def pin_backward_full_attention_autograd(lib):
    """Window = whole grid: the gradients equal torch autograd through dense
    softmax attention in fp64."""
    import torch
    grid, d = [3, 7], 8
    N = 21
    shape = (2, 1, *grid, d)
    q, k, v, do = (_randn(160 + t, shape) for t in range(4))
    dq, dk, dv = lib.backward(q, k, v, do, grid, grid, [1, 1], dtype="f32")
    qt, kt, vt = (torch.from_numpy(a.reshape(2, N, d).astype(np.float64)).requires_grad_()
                  for a in (q, k, v))
    att = torch.softmax((qt @ kt.transpose(1, 2)) / math.sqrt(d), dim=-1)
    (att @ vt).backward(torch.from_numpy(do.reshape(2, N, d).astype(np.float64)))
    for got, ref in ((dq, qt.grad), (dk, kt.grad), (dv, vt.grad)):
        np.testing.assert_allclose(got.reshape(2, N, d), ref.numpy(), atol=1e-12, rtol=0)


def pin_backward_invariants(lib):
    """Closed forms: the rows of P sum to one, so the dv of all keys sums to
    the dO of all queries; identical keys make every dq zero (each row of dZ
    sums to zero); a one-key window (w = 1) gives dv = dO and dq = dk = 0."""
    grid, window, stride, d = [6, 5], [3, 4], [2, 1], 4
    shape = (1, 2, *grid, d)
    q, k, v, do = (_randn(170 + t, shape) for t in range(4))
    dq, dk, dv = lib.backward(q, k, v, do, grid, window, stride, dtype="f32",
                              mode=["truncated", "clamped"])
    np.testing.assert_allclose(dv.sum(axis=(2, 3)), do.astype(np.float64).sum(axis=(2, 3)),
                               atol=1e-12, rtol=0)
    kc = np.broadcast_to(k[:, :, :1, :1, :], k.shape).copy()
    dq2, _, _ = lib.backward(q, kc, v, do, grid, window, stride, dtype="f32")
    np.testing.assert_allclose(dq2, 0.0, atol=1e-13, rtol=0)
    dq3, dk3, dv3 = lib.backward(q, k, v, do, grid, [1, 1], [1, 1], dtype="f32")
    np.testing.assert_allclose(dv3, do.astype(np.float64), atol=0, rtol=0)
    np.testing.assert_allclose(dq3, 0.0, atol=1e-14, rtol=0)
    np.testing.assert_allclose(dk3, 0.0, atol=1e-14, rtol=0)


def pin_backward_sampled_rows(lib):
    """The sampled-rows backward equals the full backward on every row it is
    asked for (3-D, strided, mixed modes, two heads)."""
    grid, window, stride, modes, d = [3, 5, 6], [2, 3, 4], [1, 1, 2], ["causal", "clamped",
                                                                       "truncated"], 4
    shape = (1, 2, *grid, d)
    q, k, v, do = (_randn(180 + t, shape) for t in range(4))
    dq, dk, dv = lib.backward(q, k, v, do, grid, window, stride, dtype="f32", mode=modes)
    N = 90
    rows = np.array([0, 7, 44, 89], dtype=np.int64)
    for bh in (0, 1):
        sq, sk, sv = lib.backward_sampled(q, k, v, do, grid, window, stride, bh, rows, rows[::-1],
                                          dtype="f32", mode=modes)
        np.testing.assert_allclose(sq, dq[0, bh].reshape(N, d)[rows], atol=1e-12, rtol=0)
        np.testing.assert_allclose(sk, dk[0, bh].reshape(N, d)[rows[::-1]], atol=1e-12, rtol=0)
        np.testing.assert_allclose(sv, dv[0, bh].reshape(N, d)[rows[::-1]], atol=1e-12, rtol=0)
    # Only the statistics of the queries the sampled rows read are computed:
    # key rows alone (their queries, none asked for as rows), query rows
    # alone, every row, and more threads than rows.
    every = np.arange(N, dtype=np.int64)
    none = np.zeros(0, dtype=np.int64)
    for qr, kr, th in ((none, np.array([3, 61], dtype=np.int64), 3),
                       (np.array([88, 2], dtype=np.int64), none, 5),
                       (every, every, 4), (rows, rows, 64)):
        sq, sk, sv = lib.backward_sampled(q, k, v, do, grid, window, stride, 1, qr, kr,
                                          dtype="f32", mode=modes, threads=th)
        np.testing.assert_allclose(sq, dq[0, 1].reshape(N, d)[qr], atol=1e-12, rtol=0)
        np.testing.assert_allclose(sk, dk[0, 1].reshape(N, d)[kr], atol=1e-12, rtol=0)
        np.testing.assert_allclose(sv, dv[0, 1].reshape(N, d)[kr], atol=1e-12, rtol=0)


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([float(x) for x in line.split()])
    return rows


ALL_PINS = [
    pin_window_bruteforce, pin_window_geometric_centre, pin_window_neighbourhood_metric,
    pin_window_sliding_tile, pin_window_blocked, pin_mask_bruteforce, pin_full_attention,
    pin_blocked_attention, pin_probability_rows, pin_uniform_queries, pin_single_key,
    pin_constant_values, pin_explicit_scale, pin_row_subset, pin_wsa_empty_blocks_golden,
    pin_block_counts_closed_forms, pin_ena_density_golden, pin_truncated_eq5, pin_causal_eq5,
    pin_modes_strided, pin_mode_mask_bruteforce, pin_causal_full_sdpa, pin_mode_uniform_queries,
    pin_sa_empty_blocks_golden, pin_f16_decoding, pin_e4m3_decoding,
    pin_backward_finite_differences,
    pin_backward_full_attention_autograd, pin_backward_invariants, pin_backward_sampled_rows,
    pin_dilated_window_bruteforce, pin_dilated_mask_bruteforce, pin_dilated_residue_subgrids,
    pin_dilated_backward_subgrids,
]

# The golden-file pins take a few seconds each; mutant runs use the fast ones.
FAST_PINS = [p for p in ALL_PINS if p not in (pin_wsa_empty_blocks_golden,
                                              pin_sa_empty_blocks_golden)]
