"""GPU parity on inputs built to drive the tensor-core kernel's lazy
reference-max path: the redo of a chunk whose row sum exceeds the cap, the
rescale of the accumulated O in tensor memory, and a row sum that overflows to
infinity against the stale reference.

The online softmax ("pi-Attention" section 3.1 eqs. (1)-(3), computed tile by
tile as its section 3.4 describes) keeps, per row, a reference maximum m.  The
kernel exponentiates each new chunk's scores against the m of earlier chunks
and only afterwards checks the row sum of P: if it exceeds 2^14 (or is inf /
NaN) the chunk is redone from the scores still in tensor memory against the
chunk's own maximum, and O and the running sum are rescaled by 2^(m - m_new).
On N(0, 1) inputs a later chunk never beats the running maximum by the ~14
log2 units this needs, so the ordinary parity cases never take that branch.

Construction.  Every query gets q[..., 0] = A = 16; every key gets
k[..., 0] = f(x), x its coordinate along one grid dimension p (the one whose
key-chunk extent is smallest relative to the window); the other d - 1
elements stay N(0, 1).  A score is then A f(x) / sqrt(d) plus a term of unit
spread.  A row's first effective chunk is the lowest corner of the box of
chunks its window meets in the kernel's row-major walk, so it holds only keys
with x < start_p + chunk_p; later chunks reach x = start_p + w_p - 1.
  ramp  f(x) = 8 x: the planted term grows by 128 / sqrt(d) >= 11.3 nats
        (16.3 log2 units) per unit of x, so every chunk that reaches two or
        more units of x past the row's first chunk sums far above 2^14 against
        the stale maximum and is redone, again and again along the window.
  step  f(x) = 96 for x >= L_p / 2, else 0: rows whose first chunk lies below
        the step and whose window crosses it meet a chunk whose scores beat
        the reference by 1536 / sqrt(d) >= 135 nats (> 195 log2 units), so
        2^(x - m) overflows fp32 and the row sum is +inf before the redo.
Both values are exact in bf16 and f16.  The test checks these margins on the
host from the inputs themselves (fp64 scores, an upper bound on each row's
first-chunk maximum), then compares every output element with the fp64
oracle at the parity tolerances.  Grids with full chunks only (3-D sliding
tile) and with partial chunks (2-D strided, windows not tile aligned) cover
both chunk paths, at head_dim 64 and 128, in bf16 and f16.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU machines skip the module
    pytest.skip("needs a CUDA device", allow_module_level=True)

import neighborhood_attention_b200 as na  # noqa: E402
import oracle  # noqa: E402
from gpu_parity import assert_within, compare, host_inputs, run_gpu  # noqa: E402

A = 16.0
RAMP = 8.0
STEP = 96.0
LOG2E = 1.4426950408889634

GRIDS = {
    # 3-D sliding tile: w / s odd in every dimension, so every chunk is full
    "sta3d_full": dict(grid=(8, 16, 32), window=(6, 8, 24), stride=(2, 8, 8), tile=(2, 8, 8),
                       partial=False),
    # 2-D strided: w / s = 4 is even, windows are not tile aligned -> partial chunks
    "gna2d_partial": dict(grid=(32, 48), window=(16, 16), stride=(4, 4), tile=(8, 8),
                          partial=True),
}


def _planted(c, kind, seed, p):
    q, k, v = host_inputs(c, seed)
    Lp = c["grid"][p]
    x = np.arange(Lp, dtype=np.float64)
    f = RAMP * x if kind == "ramp" else np.where(x >= Lp // 2, STEP, 0.0)
    shape = [1] * (2 + len(c["grid"]))
    shape[2 + p] = Lp
    f = np.broadcast_to(f.reshape(shape), q.shape[:-1])

    def enc(vals):
        vals = np.asarray(vals, dtype=np.float32)
        if c["dtype"] == "bf16":
            bits = vals.view(np.uint32)
            assert not (bits & 0xFFFF).any(), "planted value not exact in bf16"
            return (bits >> 16).astype(np.uint16)
        out = vals.astype(np.float16)
        assert (out.astype(np.float32) == vals).all(), "planted value not exact in f16"
        return out

    q = q.copy()
    k = k.copy()
    q[..., 0] = enc(np.full(q.shape[:-1], A))
    k[..., 0] = enc(f)
    return q, k, v


def _decode(a, dtype):
    if dtype == "bf16":
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def _margins(c, qkv, p, kbp):
    """Per query row (all heads): the largest score over the window's last slice
    along dimension p minus an upper bound of the row's first-chunk maximum
    (the scores of window keys with x_p < start_p + kbp), in log2 units."""
    grid, window, stride = c["grid"], c["window"], c["stride"]
    N = int(np.prod(grid))
    d = c["d"]
    q, k, _ = (_decode(a, c["dtype"]).reshape(-1, N, d) for a in qkv)
    coords = np.array(np.unravel_index(np.arange(N), grid))          # [ndim, N]
    starts = np.array([[oracle.window_start(grid[i], window[i], stride[i], x)
                        for x in coords[i]] for i in range(len(grid))])
    inwin = np.ones((N, N), dtype=bool)
    for i in range(len(grid)):
        xi = coords[i][None, :]
        inwin &= (xi >= starts[i][:, None]) & (xi < starts[i][:, None] + window[i])
    first = inwin & (coords[p][None, :] < starts[p][:, None] + kbp)
    last = inwin & (coords[p][None, :] == starts[p][:, None] + window[p] - 1)
    gaps = []
    for h in range(q.shape[0]):
        z = (q[h] @ k[h].T) / np.sqrt(d)
        m1 = np.where(first, z, -np.inf).max(axis=1)
        m2 = np.where(last, z, -np.inf).max(axis=1)
        gaps.append((m2 - m1) * LOG2E)
    return np.concatenate(gaps)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("kind", ["ramp", "step"])
@pytest.mark.parametrize("name", sorted(GRIDS))
def test_lazy_max_redo_and_rescale(name, kind, d, dtype):
    g = GRIDS[name]
    c = dict(B=1, heads=2, grid=g["grid"], window=g["window"], stride=g["stride"],
             tile=g["tile"], d=d, dtype=dtype)
    opts = na.make_options(kernel=na.NA_KERNEL_TC)
    plan = na.na_plan(c["grid"], c["window"], c["stride"], c["tile"], head_dim=d,
                      dtype=na.NA_F16 if dtype == "f16" else na.NA_BF16, options=opts)
    assert plan["kernel"] == "tc"
    assert (plan["units_partial"] > 0) == g["partial"], plan
    nd = len(c["grid"])
    kb = plan["kvchunk"][3 - nd:]
    p = min(range(nd), key=lambda i: (kb[i] / c["window"][i], i))
    qkv = _planted(c, kind, 4200 + d + (7 if dtype == "f16" else 0), p)
    gaps = _margins(c, qkv, p, kb[p])
    if kind == "ramp":
        # the redo fires for (almost) every row, by a wide margin
        assert np.mean(gaps > 14 + 8) >= 0.9, np.percentile(gaps, [1, 10, 50])
    else:
        # a sizeable set of rows overflows fp32 against its stale reference
        assert np.sum(gaps > 128 + 16) >= 0.05 * gaps.size, np.sum(gaps > 144)
    o, l = run_gpu(c, qkv, kernel=na.NA_KERNEL_TC)
    assert_within(c, compare(c, qkv, o, l), f"{name}/{kind}/d{d}/{dtype}")
