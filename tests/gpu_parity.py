"""Helpers for the GPU parity tests: seeded inputs on both sides, the CUDA path
through the C ABI, the fp64 oracle on the same host buffers, and the parity
bar for bf16 inputs with fp32 accumulation on N(0, 1) data:
max |out - oracle| <= 1e-2, mean |out - oracle| <= 1e-3, |lse - oracle| <= 1e-3."""
from __future__ import annotations

import numpy as np

import oracle
import seeded_inputs

TOL = {
    "bf16": dict(out_max=1e-2, out_mean=1e-3, lse_max=1e-3),
    # fp32 inputs and outputs with fp32 accumulation: rounding of ~W-term sums
    "f32": dict(out_max=5e-5, out_mean=5e-6, lse_max=5e-5),
    # f16 in and out: output rounding (half an ulp, <= 2^-10 for |out| < 2,
    # 2^-9 below 4) plus P rounded to f16 (relative 2^-11 per weight)
    "f16": dict(out_max=4e-3, out_mean=4e-4, lse_max=1e-3),
}

# The workloads: 2-D neighborhood attention (fp32 and bf16), 2-D strided
# (generalized) neighborhood attention, 3-D sliding tile attention, a 3-D
# local window covering ~30% of the sequence, and 1-D causal local attention
# over a long sequence.
CONFIGS = {
    1: dict(B=1, heads=2, grid=(16, 16), window=(5, 5), stride=(1, 1), tile=None, d=32, dtype="f32"),
    2: dict(B=4, heads=4, grid=(64, 64), window=(13, 13), stride=(1, 1), tile=None, d=64, dtype="bf16"),
    3: dict(B=2, heads=8, grid=(128, 128), window=(32, 32), stride=(8, 8), tile=(8, 8), d=64,
            dtype="bf16"),
    4: dict(B=1, heads=24, grid=(30, 48, 80), window=(18, 24, 40), stride=(6, 8, 8), tile=(6, 8, 8),
            d=128, dtype="bf16"),
    5: dict(B=2, heads=16, grid=(16, 32, 32), window=(12, 20, 20), stride=(4, 4, 4), tile=(4, 4, 4),
            d=64, dtype="bf16"),
    # 1-D causal local attention over a long sequence ("pi-Attention" section 3.2
    # eq. (5), causal case, k = 4 so w = k + 1 = 5 keys with the query itself):
    # the Medium model's 16 heads of 64 at the 32K context of its longest runs.
    6: dict(B=1, heads=16, grid=(32768,), window=(5,), stride=(1,), tile=None, d=64, dtype="bf16",
            mode=["causal"]),
}


def seed_for(cfg_id: int) -> int:
    return 1000 * cfg_id


def host_inputs(c, seed):
    return seeded_inputs.qkv(seed, c["B"], c["heads"], c["grid"], c["d"], c["dtype"])


def to_device(arr, dtype):
    import torch
    if dtype == "bf16":
        t = torch.from_numpy(arr.view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(arr)  # float32 or float16 values as they are
    return t.cuda()


def run_gpu(c, qkv_host, kernel=0, tile="cfg", qblock=None, kvchunk=None, stream=None):
    import torch
    import neighborhood_attention_b200 as na
    q, k, v = (to_device(a, c["dtype"]) for a in qkv_host)
    opts = na.make_options(kernel=kernel, qblock=qblock, kvchunk=kvchunk,
                           window_mode=c.get("mode"), ndim=len(c["grid"]), dilation=c.get("dil"))
    out, lse = na.forward(q, k, v, c["window"], c["stride"], c["tile"] if tile == "cfg" else tile,
                          options=opts, stream=stream)
    na.na_sync_status(stream)
    o = out.float().cpu().numpy().astype(np.float64)
    return o, lse.cpu().numpy().astype(np.float64)


def sample_rows(c, n_rows, seed=0):
    """Deterministic row sample: all corner and edge queries of the grid for
    the first and last head, plus uniformly drawn rows."""
    grid = c["grid"]
    N = int(np.prod(grid))
    BH = c["B"] * c["heads"]
    rng = np.random.default_rng(seed)
    picks = set()
    extremes = [sorted({0, 1, g // 2, g - 2, g - 1} & set(range(g))) for g in grid]
    import itertools
    for coord in itertools.product(*extremes):
        t = int(np.ravel_multi_index(coord, grid))
        picks.add(t)
        picks.add((BH - 1) * N + t)
    while len(picks) < n_rows:
        picks.add(int(rng.integers(0, BH * N)))
    return np.array(sorted(picks), dtype=np.int64)


def tile_tokens(grid, tile, tcoord):
    """Token indices (row-major) of the query tile at tile coordinate `tcoord`."""
    import itertools
    ranges = [range(tcoord[i] * tile[i], min((tcoord[i] + 1) * tile[i], grid[i]))
              for i in range(len(grid))]
    return np.array([np.ravel_multi_index(p, grid) for p in itertools.product(*ranges)],
                    dtype=np.int64)


def corner_edge_interior_tiles(grid, tile):
    """Tile coordinates of a 3-D tile grid sampled at its 8 corner tiles, 4 tiles
    on its edges (two coordinates at a border, one inside) and 4 interior
    tiles: the places where clamped windows differ most, and the bulk."""
    T = [grid[i] // tile[i] for i in range(3)]
    corners = [(a, b, c) for a in (0, T[0] - 1) for b in (0, T[1] - 1) for c in (0, T[2] - 1)]
    edges = [(0, 0, T[2] // 2), (T[0] - 1, T[1] - 1, T[2] // 2 - 1), (0, T[1] // 2, T[2] - 1),
             (T[0] // 2, 0, 0)]
    interior = [(T[0] // 2, T[1] // 2, T[2] // 2), (1, 1, 1), (T[0] - 2, T[1] - 2, T[2] - 2),
                (T[0] // 2, 1, T[2] - 3)]
    return corners, edges, interior


def compare(c, qkv_host, out_gpu, lse_gpu, rows=None):
    """Oracle on the same host buffers; returns (max|dout|, mean|dout|, max|dlse|)."""
    q, k, v = qkv_host
    d = c["d"]
    if rows is None:
        ref_o, ref_l = oracle.forward(q, k, v, c["grid"], c["window"], c["stride"], dtype=c["dtype"],
                                      mode=c.get("mode"), dilation=c.get("dil"))
        go = out_gpu
        gl = lse_gpu
        ref_o = ref_o.reshape(go.shape)
        ref_l = ref_l.reshape(gl.shape)
    else:
        ref_o, ref_l = oracle.forward(q, k, v, c["grid"], c["window"], c["stride"], dtype=c["dtype"],
                                      rows=rows, mode=c.get("mode"), dilation=c.get("dil"))
        go = out_gpu.reshape(-1, d)[rows]
        gl = lse_gpu.reshape(-1)[rows]
    do = np.abs(go - ref_o)
    dl = np.abs(gl - ref_l)
    assert np.isfinite(go).all() and np.isfinite(gl).all(), "non-finite GPU output"
    return float(do.max()), float(do.mean()), float(dl.max())


def assert_within(c, errs, label=""):
    tol = TOL[c["dtype"]]
    omax, omean, lmax = errs
    assert omax <= tol["out_max"], f"{label} max|dout|={omax:.3e} > {tol['out_max']}"
    assert omean <= tol["out_mean"], f"{label} mean|dout|={omean:.3e} > {tol['out_mean']}"
    assert lmax <= tol["lse_max"], f"{label} max|dlse|={lmax:.3e} > {tol['lse_max']}"
