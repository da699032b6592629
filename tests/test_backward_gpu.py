"""GPU parity of the backward pass: dq, dk, dv from the CUDA kernels (through
the C ABI, after the CUDA forward produced out and lse) against the fp64
oracle's gradients on identical seeded inputs, element by element.

Bar, from the arithmetic: 16-bit gradients are rounded once to the input
type (half an ulp, 2^-9 relative for bf16, 2^-12 for f16); on the tensor-core
path dS is also rounded to the input type as the operand of dq's product (as
P is in the forward), each of the window's terms carrying that relative
error; and the forward's 16-bit out enters D_i = <dO_i, out_i>.  fp32
accumulation adds far less.  So for bf16 / f16
max |g - oracle| <= 2^-7 max|oracle| + 4e-3 and mean <= 2^-8 mean|oracle| + 2e-4;
fp32 inputs (CUDA cores only): max <= 1e-4 max(1, max|oracle|), mean <= 1e-5."""
import zlib

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU machines skip the module
    pytest.skip("needs a CUDA device", allow_module_level=True)

import neighborhood_attention_b200 as na  # noqa: E402
import oracle  # noqa: E402
import seeded_inputs  # noqa: E402
from gpu_parity import to_device  # noqa: E402


def _case(grid, window, stride, d, dtype="bf16", B=1, heads=2, mode=None, tile=None, dil=None):
    return dict(B=B, heads=heads, grid=tuple(grid), window=tuple(window), stride=tuple(stride),
                d=d, dtype=dtype, mode=mode, tile=tile, dil=dil)


CASES = {
    "na2d_ragged_d64": _case((21, 27), (7, 5), (1, 1), 64),
    "na2d_d128": _case((13, 17), (5, 7), (1, 1), 128),
    "gna2d_strided": _case((24, 20), (12, 8), (4, 2), 64),
    "sta3d_small": _case((6, 8, 16), (6, 8, 8), (2, 4, 4), 64, tile=(2, 4, 4)),
    "na1d_long": _case((700,), (65,), (1,), 64),
    "causal1d": _case((500,), (97,), (1,), 128, mode=["causal"]),
    "truncated_mixed3d": _case((5, 9, 11), (3, 5, 7), (1, 2, 1), 32,
                               mode=["truncated", "causal", "clamped"], B=2, heads=1),
    "full_attention": _case((12, 16), (12, 16), (1, 1), 64),
    "fp32_d32": _case((16, 16), (5, 5), (1, 1), 32, dtype="f32", heads=3),
    "f16_d64": _case((18, 22), (7, 9), (2, 1), 64, dtype="f16"),
    "sta3d_medium_d128": _case((6, 16, 40), (6, 12, 24), (2, 4, 8), 128, tile=(2, 4, 8)),
    # about ten chunks per block at head_dim 64: the four-stage slots of both
    # gradient kernels go through several rounds
    "sta3d_medium_d64": _case((6, 16, 40), (6, 12, 24), (2, 4, 8), 64, tile=(2, 4, 8)),
    # dilated windows (residue classes of different lengths)
    "dilated2d_d64": _case((23, 17), (5, 4), (1, 2), 64, dil=(3, 2),
                           mode=["clamped", "truncated"]),
    "dilated1d_causal_d128": _case((401,), (33,), (1,), 128, dil=(4,), mode=["causal"]),
    "dilated3d_f32": _case((6, 9, 10), (3, 3, 4), (1, 1, 2), 32, dtype="f32", dil=(2, 3, 2)),
}


def _run(c, seed, kernel=None):
    shape = (c["B"], c["heads"], *c["grid"], c["d"])
    q, k, v = seeded_inputs.qkv(seed, c["B"], c["heads"], c["grid"], c["d"], c["dtype"])
    gen = {"f32": seeded_inputs.normal_f32, "bf16": seeded_inputs.normal_bf16_bits,
           "f16": seeded_inputs.normal_f16}[c["dtype"]]
    do = gen(seed + 7, shape, threads=1)
    qd, kd, vd, dod = (to_device(a, c["dtype"]) for a in (q, k, v, do))
    opts = na.make_options(window_mode=c["mode"], ndim=len(c["grid"]), dilation=c["dil"])
    out, lse = na.forward(qd, kd, vd, c["window"], c["stride"], c["tile"], options=opts)
    bopts = na.make_options(window_mode=c["mode"], ndim=len(c["grid"]), dilation=c["dil"],
                            kernel=kernel if kernel is not None else na.NA_KERNEL_AUTO)
    dq, dk, dv = na.backward(qd, kd, vd, out, lse, dod, c["window"], c["stride"], c["tile"],
                             options=bopts)
    na.na_sync_status()
    got = [t.float().cpu().numpy().astype(np.float64) for t in (dq, dk, dv)]
    ref = oracle.backward(q, k, v, do, c["grid"], c["window"], c["stride"], dtype=c["dtype"],
                          mode=c["mode"], dilation=c["dil"])
    return got, ref


def _assert_close(c, got, ref, label, names=("dq", "dk", "dv")):
    for name, g, r in zip(names, got, ref):
        assert np.isfinite(g).all(), f"{label} {name}: non-finite"
        err = np.abs(g - r)
        if c["dtype"] == "f32":
            tmax, tmean = 1e-4 * max(1.0, np.abs(r).max()), 1e-5
        else:
            tmax = 2.0 ** -7 * np.abs(r).max() + 4e-3
            tmean = 2.0 ** -8 * np.abs(r).mean() + 2e-4
        assert err.max() <= tmax, f"{label} {name}: max|err|={err.max():.3e} > {tmax:.3e}"
        assert err.mean() <= tmean, f"{label} {name}: mean|err|={err.mean():.3e} > {tmean:.3e}"


@pytest.mark.parametrize("name", sorted(CASES))
def test_backward_parity(name):
    """The default path: tensor-core dQ for bf16 / f16 with head_dim 64 or 128,
    CUDA-core kernels otherwise."""
    c = CASES[name]
    got, ref = _run(c, seed=zlib.crc32(name.encode()) % 100000)
    _assert_close(c, got, ref, name)


@pytest.mark.parametrize("name", ["na2d_ragged_d64", "causal1d", "sta3d_small", "f16_d64",
                                  "dilated2d_d64"])
def test_backward_parity_cuda_cores(name):
    """The same cases with every backward kernel on the CUDA cores."""
    c = CASES[name]
    got, ref = _run(c, seed=zlib.crc32(name.encode()) % 100000, kernel=na.NA_KERNEL_SIMT)
    _assert_close(c, got, ref, name + "/simt")


def test_backward_deterministic():
    c = CASES["gna2d_strided"]
    a, _ = _run(c, seed=31)
    b, _ = _run(c, seed=31)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_backward_tensor_core_selector_needs_16_bit():
    c = CASES["fp32_d32"]
    q = torch.zeros((1, 1, *c["grid"], 64), dtype=torch.float32, device="cuda")
    lse = torch.zeros(q.shape[:-1], dtype=torch.float32, device="cuda")
    with pytest.raises(na.NaError) as e:
        na.backward(q, q, q, q, lse, q, c["window"], options=na.make_options(kernel=na.NA_KERNEL_TC))
    assert e.value.status == na.NA_ERR_UNSUPPORTED


def _sample_keys(grid, n, seed):
    """Corner and edge tokens of the grid plus uniform draws (token indices)."""
    import itertools
    N = int(np.prod(grid))
    extremes = [sorted({0, 1, g // 2, g - 2, g - 1} & set(range(g))) for g in grid]
    picks = {int(np.ravel_multi_index(c, grid)) for c in itertools.product(*extremes)}
    rng = np.random.default_rng(seed)
    while len(picks) < n:
        picks.add(int(rng.integers(0, N)))
    return np.array(sorted(picks), dtype=np.int64)


def _full_size_grads(c, seed):
    shape = (c["B"], c["heads"], *c["grid"], c["d"])
    q, k, v = seeded_inputs.qkv(seed, c["B"], c["heads"], c["grid"], c["d"], c["dtype"])
    do = seeded_inputs.normal_bf16_bits(seed + 7, shape)
    qd, kd, vd, dod = (to_device(a, c["dtype"]) for a in (q, k, v, do))
    out, lse = na.forward(qd, kd, vd, c["window"], c["stride"], c["tile"])
    dq, dk, dv = na.backward(qd, kd, vd, out, lse, dod, c["window"], c["stride"], c["tile"])
    na.na_sync_status()
    return (q, k, v, do), (dq, dk, dv), dod


def _rows_of(t, b, h, N, d, rows):
    return (t[b, h].reshape(N, d)[torch.from_numpy(rows).cuda()].float().cpu().numpy()
            .astype(np.float64))


def test_backward_sliding_tile_full_size_tiles_of_every_head():
    """The 3-D sliding tile workload (24 heads, 30 x 48 x 80, tile 6 x 8 x 8,
    window 18 x 24 x 40, d 128) in the benchmark's launch configuration.
    In every head: dq of 8 rows from each of the 8 corner, 4 edge and 4
    interior tiles, and dk, dv of every key of one whole tile (heads 0-7 the
    8 corner tiles, 8-11 the edge tiles, 12-13 two interior tiles, 14-23 the
    corner tiles again), against the oracle's sampled backward, which computes
    the softmax statistics of exactly the queries those rows read.  Every head
    also keeps sum_j dv_j = sum_i dO_i (each row of P sums to one) over all
    115,200 keys; its bar is 8 times the root-sum-square of the two rounding
    steps that perturb it: dv_j to bf16 (2^-9 |dv_j|) and, per query, the
    window's P rounded to bf16 as the operand of dV (2^-9 P_ij per key,
    averaging over the W keys of the window)."""
    c = _case((30, 48, 80), (18, 24, 40), (6, 8, 8), 128, heads=24, tile=(6, 8, 8))
    from gpu_parity import corner_edge_interior_tiles, tile_tokens
    host, (dq, dk, dv), dod = _full_size_grads(c, 9100)
    q, k, v, do = host
    N = int(np.prod(c["grid"]))
    W = int(np.prod(c["window"]))
    corners, edges, interior = corner_edge_interior_tiles(c["grid"], c["tile"])
    qrows = np.concatenate([tile_tokens(c["grid"], c["tile"], t)[::48]
                            for t in corners + edges + interior])
    key_tiles = corners + edges + interior[:2] + corners[::-1] + edges[:2]
    assert len(key_tiles) == c["heads"]
    # sum over keys of dv, per head, in fp64 on the device
    sum_dv = dv.double().reshape(c["heads"], N, c["d"]).sum(dim=1)
    sum_do = dod.double().reshape(c["heads"], N, c["d"]).sum(dim=1)
    rss = torch.sqrt((dv.double() ** 2).reshape(c["heads"], N, c["d"]).sum(dim=1)
                     + (dod.double() ** 2).reshape(c["heads"], N, c["d"]).sum(dim=1) / W)
    assert ((sum_dv - sum_do).abs() <= 8 * 2.0 ** -9 * rss).all(), \
        float(((sum_dv - sum_do).abs() / rss).max())
    for h in range(c["heads"]):
        krows = tile_tokens(c["grid"], c["tile"], key_tiles[h])
        rq, rk, rv = oracle.backward_sampled(q, k, v, do, c["grid"], c["window"], c["stride"], h,
                                             qrows, krows, dtype="bf16")
        got_q = _rows_of(dq, 0, h, N, c["d"], qrows)
        got_k, got_v = (_rows_of(t, 0, h, N, c["d"], krows) for t in (dk, dv))
        _assert_close(c, [got_q], [rq], f"head {h}", names=("dq",))
        _assert_close(c, [got_k, got_v], [rk, rv], f"head {h} tile {key_tiles[h]}",
                      names=("dk", "dv"))


def test_backward_local3d_full_size_sampled():
    """The 3-D local workload (32 heads, 16 x 32 x 32, window 12 x 20 x 20,
    stride 4, d 64) in the benchmark's launch configuration: dq, dk, dv of
    sampled rows (grid corners, edges and uniform draws) of the first and last
    (batch, head) slice against the oracle's sampled backward."""
    c = _case((16, 32, 32), (12, 20, 20), (4, 4, 4), 64, B=2, heads=16, tile=(4, 4, 4))
    host, (dq, dk, dv), _ = _full_size_grads(c, 9200)
    q, k, v, do = host
    BH = c["B"] * c["heads"]
    N = int(np.prod(c["grid"]))
    rows = _sample_keys(c["grid"], 96, 9200)
    for bh in (0, BH - 1):
        rq, rk, rv = oracle.backward_sampled(q, k, v, do, c["grid"], c["window"], c["stride"], bh,
                                             rows, rows, dtype="bf16")
        b, h = divmod(bh, c["heads"])
        got = [_rows_of(t, b, h, N, c["d"], rows) for t in (dq, dk, dv)]
        _assert_close(c, got, (rq, rk, rv), f"local3d bh={bh}")


def _random_bwd_case(seed):
    """A seeded random backward problem: 1-3 dimensions, any window mode and
    stride, bf16 or f16 at head_dim 64 / 128 (tensor cores) or fp32 at 32."""
    rng = np.random.default_rng(seed)
    nd = int(rng.integers(1, 4))
    cap = {1: 600, 2: 30, 3: 10}[nd]
    grid = [int(rng.integers(3, cap + 1)) for _ in range(nd)]
    window = [int(rng.integers(1, g + 1)) for g in grid]
    stride = [int(rng.integers(1, w + 1)) for w in window]
    mode = [["clamped", "truncated", "causal"][int(rng.integers(0, 3))] for _ in range(nd)]
    kind = int(rng.integers(0, 3))
    d, dtype = [(64, "bf16"), (128, "f16"), (32, "f32")][kind]
    return _case(grid, window, stride, d, dtype=dtype, heads=int(rng.integers(1, 3)), mode=mode)


@pytest.mark.parametrize("seed", range(8))
def test_backward_random_problems(seed):
    """Seeded random problems through the default backward path, dq / dk / dv
    against the oracle's gradients."""
    c = _random_bwd_case(6100 + seed)
    got, ref = _run(c, seed=6200 + seed)
    _assert_close(c, got, ref, f"random {seed}: {c}")
