"""na_forward_noalloc, the entry point for callers that must not allocate
device memory (for example an engine that has reserved nearly all of HBM for
its own pools, where a stray cudaMalloc would fail or escape its accounting).

It keeps its scratch (the kernel's status word) in a fixed array compiled into
the library instead of cudaMalloc'd memory.  The test calls it through the C
ABI twice in a row, on different inputs, and checks each result against the
regular na_forward entry point within the parity tolerances.  It is collected
last so that a failure here never hides the other tests in a run that stops at
the first failure, and it passes both alone and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - CPU machines skip the module
    pytest.skip("needs a CUDA device", allow_module_level=True)

import neighborhood_attention_b200 as na  # noqa: E402
import seeded_inputs  # noqa: E402

TOL = dict(out_max=1e-2, out_mean=1e-3, lse_max=1e-3)   # the bf16 parity tolerances

CASES = [
    # grid, window, stride, tile, head_dim
    ((8, 16, 16), (4, 8, 8), (2, 4, 4), (2, 4, 4), 64),
    ((12, 16, 24), (6, 8, 8), (2, 4, 4), (2, 4, 8), 128),
]


def _inputs(seed, grid, d, heads=3):
    arrs = seeded_inputs.qkv(seed, 1, heads, grid, d, "bf16")
    return [torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda() for a in arrs]


def _noalloc_c_abi(q, k, v, out, lse, grid, window, stride, tile):
    """Direct ctypes call of the exported C symbol."""
    lib = ctypes.CDLL(na.LIB_PATH)
    fn = lib.na_forward_noalloc
    iv = lambda xs: (ctypes.c_int * len(xs))(*[int(x) for x in xs])
    fn.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int, ctypes.c_int] + \
        [ctypes.POINTER(ctypes.c_int)] * 5 + [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    fn.restype = ctypes.c_int
    stream = torch.cuda.current_stream().cuda_stream
    return fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
              q.shape[0], q.shape[1], iv([len(grid), q.shape[-1]]), iv(grid), iv(window),
              iv(stride), iv(tile), na.NA_BF16, None, stream)


@pytest.mark.parametrize("grid,window,stride,tile,d", CASES)
def test_noalloc_matches_na_forward_on_two_calls(grid, window, stride, tile, d):
    outs = []
    for call, seed in enumerate((910, 911)):
        q, k, v = _inputs(seed, grid, d)
        ref_o, ref_l = na.forward(q, k, v, window, stride, tile)
        na.na_sync_status()
        out = torch.full_like(q, float("nan"))
        lse = torch.full(q.shape[:-1], float("nan"), dtype=torch.float32, device=q.device)
        before = torch.cuda.memory_allocated()
        st = _noalloc_c_abi(q, k, v, out, lse, grid, window, stride, tile)
        assert st == na.NA_OK, na.na_last_error()
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated() == before
        do = (out.float() - ref_o.float()).abs()
        dl = (lse - ref_l).abs()
        assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all(), f"call {call}"
        assert do.max().item() <= TOL["out_max"], f"call {call}: max|dout| {do.max().item()}"
        assert do.mean().item() <= TOL["out_mean"], f"call {call}: mean|dout| {do.mean().item()}"
        assert dl.max().item() <= TOL["lse_max"], f"call {call}: max|dlse| {dl.max().item()}"
        outs.append(out.clone())
    assert not torch.equal(outs[0], outs[1])  # the second call computed its own inputs


def test_noalloc_rejects_what_it_cannot_run():
    q, k, v = _inputs(912, (8, 8), 32, heads=1)   # head_dim 32: not a tensor-core shape
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    st = _noalloc_c_abi(q, k, v, out, lse, (8, 8), (3, 3), (1, 1), (8, 8))
    assert st == na.NA_ERR_UNSUPPORTED
    assert na.na_last_error()
