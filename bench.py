"""Benchmark of the forward pass on the 3-D sliding tile attention workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (one step = one forward pass over one batch): B=1, heads=24,
head_dim=128, grid T x H x W = 30 x 48 x 80 (115,200 tokens), tile 6x8x8,
window 18x24x40 (3x3x5 tiles), stride = tile, bf16 inputs drawn N(0, 1) from
fixed seeds.  Metric: effective TFLOP/s = 4 * d * B * heads * N * prod(window)
/ time, i.e. only the (query, key) pairs inside windows count.

Our arm times the tensor-core kernel through the C ABI with inputs resident in
HBM (q, k, v total 2.1 GB, larger than the 126 MB L2, so no flush is needed),
plus an end-to-end figure with pinned-host inputs copied in and outputs copied
out inside the timed region (pipelined across steps: the copies of one step
overlap the compute of its neighbours, two device buffer sets).  The reference arm (--impl reference) times the
fp64 CPU oracle on a bounded sample of query rows on the host cores.

With N > 1 (torchrun), every rank runs its own replica of the workload (weak
scaling; the problem has no exchange step), the timed region is bracketed by
barriers, and the time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "effective TFLOP/s and % of B200 bf16 tensor peak, 3D sliding-tile attn fwd"
WORKLOAD = dict(workload="3D sliding tile attention fwd", B=1, heads=24, head_dim=128,
                grid=[30, 48, 80], tile=[6, 8, 8], window=[18, 24, 40], stride=[6, 8, 8],
                dtype="bf16")
# The other workloads of the parity suite, selectable with --config (the
# default, 4, is the one the metric is quoted on).
WORKLOADS = {
    1: dict(workload="2D neighborhood attention fwd, fp32", B=1, heads=2, head_dim=32,
            grid=[16, 16], tile=None, window=[5, 5], stride=[1, 1], dtype="f32"),
    2: dict(workload="2D neighborhood attention fwd", B=4, heads=4, head_dim=64,
            grid=[64, 64], tile=None, window=[13, 13], stride=[1, 1], dtype="bf16"),
    3: dict(workload="2D generalized neighborhood attention fwd", B=2, heads=8, head_dim=64,
            grid=[128, 128], tile=[8, 8], window=[32, 32], stride=[8, 8], dtype="bf16"),
    4: WORKLOAD,
    5: dict(workload="3D local attention at ~30% density fwd", B=2, heads=16, head_dim=64,
            grid=[16, 32, 32], tile=[4, 4, 4], window=[12, 20, 20], stride=[4, 4, 4],
            dtype="bf16"),
    # 1-D causal local attention over a long sequence: each token sees itself
    # and the k = 4 before it (w = k + 1), 16 heads of 64, 32K tokens.
    6: dict(workload="1D causal local attention, long sequence fwd", B=1, heads=16, head_dim=64,
            grid=[32768], tile=None, window=[5], stride=[1], window_mode=["causal"],
            dtype="bf16"),
}
SEED = 4000
FALLBACK_PEAK_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = ["neighborhood_attention_b200/csrc/na_fwd_sm100.cu",
                  "neighborhood_attention_b200/csrc/na_ptx.cuh",
                  "neighborhood_attention_b200/csrc/na_sched.cuh"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "na_fwd_tc_sta3d_traffic.txt")
TRAFFIC_APPLIES = True     # the traffic file covers only the default 24-head workload
L2_BYTES = 126 * 10**6
DENSE_STEPS = 3
FLUSH_BYTES = 256 * 2**20
RUNS = 10                 # repeated runs for the median / min
FP8_PER_BF16 = 2.0        # nominal dense tensor rate of 8-bit vs 16-bit operands
REPEAT_BUDGET_S = 8.0     # launches per run sized to about this much kernel time in all


def flops_per_step(useful_pairs, w=None):
    """4 d FLOPs per attended (query, key) pair of one head, times the heads.
    useful_pairs = N * prod(window) for clamped windows (every query sees a
    full window); cut (truncated / causal) windows see fewer keys at the
    borders, so the count comes from the scheduler's per-dimension sums."""
    w = WORKLOAD if w is None else w
    return 4.0 * w["head_dim"] * w["B"] * w["heads"] * useful_pairs


def min_hbm_bytes(w=None):
    """Algorithmic HBM bytes of one forward: q, k, v read and out written once
    (d elements each per token), lse written once (4 bytes per token)."""
    w = WORKLOAD if w is None else w
    tokens = w["B"] * w["heads"] * int(np.prod(w["grid"]))
    if w["dtype"] == "e4m3":      # 1-byte q, k, v; bf16 out
        return tokens * ((3 * 1 + 2) * w["head_dim"] + 4)
    elt = 4 if w["dtype"] == "f32" else 2
    return tokens * (4 * w["head_dim"] * elt + 4)


def options_for(na, w=None):
    w = WORKLOAD if w is None else w
    if not w.get("window_mode"):
        return None
    return na.make_options(window_mode=w["window_mode"], ndim=len(w["grid"]))


def kernel_hash():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def read_traffic():
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    try:
        kv = {}
        with open(TRAFFIC_FILE) as f:
            for line in f:
                parts = line.split()
                if len(parts) == 2 and not line.startswith("#"):
                    kv[parts[0]] = parts[1]
        if kv.get("kernel_hash") == kernel_hash():
            return float(kv["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        pass
    return None


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", 0) or 0), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_PEAK_TFLOPS, 0.0, "fallback"


def read_hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self, windows=()):
        """Median SM clock and throttle reasons over the samples taken inside
        the given (start, end) wall-clock windows (all samples if none)."""
        import datetime
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                except ValueError:
                    ts = None
                if windows and (ts is None or not any(a <= ts <= b for a, b in windows)):
                    continue
                try:
                    sm.append(float(parts[2]))
                    smax.append(float(parts[3]))
                except ValueError:
                    continue
                for n, val in zip(names, parts[6:10]):
                    if val.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- CPU side --
def workload_rows(w=None):
    """Query rows of a workload: B * heads * grid tokens."""
    w = WORKLOAD if w is None else w
    return int(w["B"] * w["heads"] * np.prod(w["grid"]))


def oracle_sample_rows(n_rows, seed=1):
    """n_rows distinct query rows drawn uniformly (sorted); every row when the
    workload has no more than n_rows."""
    total = workload_rows()
    if n_rows >= total:
        return np.arange(total, dtype=np.int64)
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(total, size=n_rows, replace=False)).astype(np.int64)


def host_qkv():
    import seeded_inputs
    w = WORKLOAD
    return seeded_inputs.qkv(SEED, w["B"], w["heads"], w["grid"], w["head_dim"], w["dtype"])


def time_oracle(qkv, n_rows, threads):
    import oracle
    w = WORKLOAD
    rows = oracle_sample_rows(n_rows)
    t0 = time.perf_counter()
    oracle.forward(*qkv, w["grid"], w["window"], w["stride"], dtype=w["dtype"], rows=rows,
                   threads=threads, mode=w.get("window_mode"))
    dt = time.perf_counter() - t0
    flops = 4.0 * w["head_dim"] * sampled_pairs(rows)
    return flops / dt / 1e12, dt


def sampled_pairs(rows):
    """Attended (query, key) pairs of the sampled rows, from the oracle's own
    window rule (the product over dimensions of each window's length)."""
    import oracle
    w = WORKLOAD
    grid = w["grid"]
    N = int(np.prod(grid))
    modes = w.get("window_mode") or ["clamped"] * len(grid)
    coords = np.unravel_index(np.asarray(rows) % N, grid)
    lens = []
    for d, L in enumerate(grid):
        cache = {}
        per = []
        for i in coords[d].tolist():
            if i not in cache:
                lo, hi = oracle.window(L, w["window"][d], w["stride"][d], modes[d], i)
                cache[i] = hi - lo
            per.append(cache[i])
        lens.append(np.array(per, dtype=np.int64))
    return int(np.sum(np.prod(np.stack(lens), axis=0)))


def cpu_baseline(qkv, target_s=15.0):
    threads = os.cpu_count() or 1
    probe = max(64, threads * 8)
    _, dt = time_oracle(qkv, probe, threads)
    n = min(workload_rows(), int(min(200000, max(probe, probe * target_s / max(dt, 1e-3)))))
    val, dt = time_oracle(qkv, n, threads)
    return {"value": val, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} query rows drawn uniformly from the workload's {workload_rows()} "
                      f"(fp64 dense-mask oracle, {dt:.1f} s)"}


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    qkv = host_qkv()
    threads = os.cpu_count() or 1
    probe = max(64, threads * 8)
    _, dt = time_oracle(qkv, probe, threads)
    # each step a bounded sample sized so that warm-up + timed steps end within minutes
    budget = 120.0 / max(1, args.steps + args.warmup)
    n = min(workload_rows(), int(max(probe, probe * min(budget, 20.0) / max(dt, 1e-3))))
    for _ in range(args.warmup):
        time_oracle(qkv, n, threads)
    tot = 0.0
    for _ in range(args.steps):
        _, dt = time_oracle(qkv, n, threads)
        tot += dt
    flops = 4.0 * WORKLOAD["head_dim"] * sampled_pairs(oracle_sample_rows(n)) * args.steps
    value = flops / tot / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * tot / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(WORKLOAD, sample_rows_per_step=n),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"{n} query rows per step"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------ rank logic --
def max_over_ranks(values, world, device):
    """Element-wise maximum of a list of floats over all ranks (identity when world == 1)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_tflops(flops_per_rank_step, steps, world, max_ms):
    """Whole-job throughput: the work every rank did (each rank runs one replica
    of the workload per step) over the slowest rank's time."""
    return flops_per_rank_step * steps * world / (max_ms / 1e3) / 1e12


# ---------------------------------------------------------------- GPU side --
FP32_FMA_PER_CLK_SM = 128      # fp32 FMA lanes per SM per clock (B200)
NUM_SM = 148


def run_backward(args, rank, world, local_rank):
    """The backward pass (na_backward: dq, dk, dv) on the selected workload:
    one step = one call (row delta, then the dq and dk / dv kernels -- on the
    tensor cores for bf16 / f16 with head_dim 64 or 128); the forward's out
    and lse are produced once before timing.  Effective TFLOP/s counts 10 * d
    FLOPs per attended (query, key) pair (five products of 2 d: scores, dP, dV,
    dQ, dK; the two kernels each recompute scores and dP, which is not
    counted), against the measured dense bf16 peak -- or, when the CUDA-core
    kernels run, the fp32 FMA peak at the sampled clock."""
    import torch
    import torch.distributed as dist
    import neighborhood_attention_b200 as na

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = WORKLOAD
    qkv_host = host_qkv()
    if w["dtype"] == "bf16":
        tensors = [torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) for a in qkv_host]
    else:
        tensors = [torch.from_numpy(a) for a in qkv_host]
    q, k, v = (t.to(dev) for t in tensors)
    g = torch.Generator(device=dev).manual_seed(SEED + 11)
    dout = torch.randn(q.shape, generator=g, device=dev, dtype=torch.float32).to(q.dtype)
    stream = torch.cuda.current_stream(dev)
    opts = options_for(na)
    out, lse = na.forward(q, k, v, w["window"], w["stride"], w["tile"], options=opts,
                          stream=stream)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    delta = torch.empty(lse.shape, dtype=torch.float32, device=dev)

    def step():
        na.na_backward(q, k, v, out, dout, lse, dq, dk, dv, delta, w["window"], w["stride"],
                       w["tile"], options=opts, stream=stream)

    for _ in range(args.warmup):
        step()
    na.na_sync_status(stream)
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(1.0)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    w0 = time.time()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    w1 = time.time()
    clocks = sampler.stop(windows=[(w0, w1)])
    if world > 1:
        dist.barrier()
    na.na_sync_status(stream)
    (total_ms,) = max_over_ranks([e0.elapsed_time(e1)], world, dev)
    plan = na.na_plan(w["grid"], w["window"], w["stride"], w["tile"], w["head_dim"],
                      {"bf16": na.NA_BF16, "f16": na.NA_F16, "f32": na.NA_F32,
                       "e4m3": na.NA_E4M3}[w["dtype"]],
                      options=opts)
    flops = 10.0 * w["head_dim"] * w["B"] * w["heads"] * plan["useful_pairs"]
    value = flops * args.steps * world / (total_ms / 1e3) / 1e12
    tensor = w["dtype"] in ("bf16", "f16") and w["head_dim"] in (64, 128)
    if tensor:
        peak, _, peak_kind = read_peaks()
        peak_kind = (f"{peak_kind} burst bf16 (MEASURED_PEAKS.json)" if peak_kind == "measured"
                     else "fallback")
    else:
        mhz = clocks.get("sm_mhz") or clocks.get("sm_max_mhz") or 1965.0
        peak = 2.0 * FP32_FMA_PER_CLK_SM * NUM_SM * mhz * 1e6 / 1e12
        peak_kind = "derived: 148 SM x 128 fp32 FMA/clk x 2 FLOP x sampled SM clock"
    achieved = value / world
    if rank != 0:
        return 0
    line = {
        "metric": f"effective TFLOP/s, backward (dq, dk, dv), {w['workload']}",
        "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w["dtype"], "data": "synthetic",
        "config": dict(w, direction="backward",
                       kernels="tcgen05 dq and dk/dv" if tensor else "CUDA-core (fp32 FMA)"),
        "roofline": {"bound": "tensor" if tensor else "alu", "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak, "traffic": None,
                     "peak_kind": peak_kind},
        "gpu_launches": 3 * args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import neighborhood_attention_b200 as na

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = WORKLOAD
    qkv_host = host_qkv()
    if w["dtype"] == "bf16":
        pinned = [torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory()
                  for a in qkv_host]
    elif w["dtype"] == "e4m3":
        pinned = [torch.from_numpy(a).view(torch.float8_e4m3fn).pin_memory() for a in qkv_host]
    else:
        pinned = [torch.from_numpy(a).pin_memory() for a in qkv_host]
    q, k, v = (t.to(dev) for t in pinned)
    out = torch.empty(q.shape, dtype=na.out_dtype(q), device=dev)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=dev)
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    lse_host = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    stream = torch.cuda.current_stream(dev)
    opts = options_for(na)

    def step():
        na.na_forward_ex(q, k, v, out, lse, w["window"], w["stride"], w["tile"], options=opts,
                         stream=stream)

    # Inputs that do not clearly exceed L2 would stay cached from one step to
    # the next: then L2 is flushed (a 256 MB write) before every timed step and
    # the time is the sum of per-step event pairs, which exclude the flush.
    h2d = sum(t.numel() * t.element_size() for t in pinned)
    flush = h2d < 2 * L2_BYTES
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if flush else None

    def flush_l2(i):
        if flush:
            flush_buf.fill_(i & 0xFF)

    for _ in range(args.warmup):
        step()
    na.na_sync_status(stream)

    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(1.0)   # let nvidia-smi start sampling before the timed region
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    w0 = time.time()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        flush_l2(i)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    w1 = time.time()
    if world > 1:
        dist.barrier()
    na.na_sync_status(stream)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = float(np.sum(step_ms)) if flush else t_start.elapsed_time(t_end)
    per_launch_ms = float(np.mean(step_ms))

    # end to end through the public API: pinned host -> device, forward, device -> host
    d2h = out_host.numel() * out_host.element_size() + lse_host.numel() * lse_host.element_size()

    def e2e_step():
        q.copy_(pinned[0], non_blocking=True)
        k.copy_(pinned[1], non_blocking=True)
        v.copy_(pinned[2], non_blocking=True)
        step()
        out_host.copy_(out, non_blocking=True)
        lse_host.copy_(lse, non_blocking=True)

    # Pipelined form (inputs larger than L2): two device buffer sets and
    # separate copy streams, so step i+1's host -> device copy and step i-1's
    # device -> host copy run while step i computes.  Every step still copies
    # its own inputs in and its own results out inside the timed region.
    pipelined = not flush
    if pipelined:
        bufs = [(q, k, v, out, lse)] + [
            tuple(torch.empty_like(t) for t in (q, k, v, out, lse))]
        s_in = torch.cuda.Stream(dev)
        s_out = torch.cuda.Stream(dev)

        def e2e_run(nsteps, first_ev=None, last_ev=None):
            h2d_done = [torch.cuda.Event() for _ in range(nsteps)]
            comp_done = [torch.cuda.Event() for _ in range(nsteps)]
            d2h_done = [torch.cuda.Event() for _ in range(nsteps)]
            if first_ev is not None:
                first_ev.record(s_in)
            for i in range(nsteps):
                bq, bk, bv, bo, bl = bufs[i % 2]
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(comp_done[i - 2])   # inputs of buffer i%2 consumed
                    bq.copy_(pinned[0], non_blocking=True)
                    bk.copy_(pinned[1], non_blocking=True)
                    bv.copy_(pinned[2], non_blocking=True)
                    h2d_done[i].record(s_in)
                stream.wait_event(h2d_done[i])
                if i >= 2:
                    stream.wait_event(d2h_done[i - 2])      # outputs of buffer i%2 copied out
                na.na_forward_ex(bq, bk, bv, bo, bl, w["window"], w["stride"], w["tile"],
                                 options=opts, stream=stream)
                comp_done[i].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(comp_done[i])
                    out_host.copy_(bo, non_blocking=True)
                    lse_host.copy_(bl, non_blocking=True)
                    d2h_done[i].record(s_out)
            if last_ev is not None:
                last_ev.record(s_out)

        e2e_run(min(args.warmup, 2))
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        w2 = time.time()
        e2e_run(args.steps, e0, e1)
        torch.cuda.synchronize()
        w3 = time.time()
        e2e_ms = e0.elapsed_time(e1)
    else:
        for _ in range(min(args.warmup, 2)):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.steps)]
        w2 = time.time()
        for i in range(args.steps):
            flush_l2(i)
            e_ev[i][0].record(stream)
            e2e_step()
            e_ev[i][1].record(stream)
        torch.cuda.synchronize()
        w3 = time.time()
        e2e_ms = float(np.sum([a.elapsed_time(b) for a, b in e_ev]))
    clocks = sampler.stop(windows=[(w0, w1), (w2, w3)])
    if world > 1:
        dist.barrier()
    na.na_sync_status(stream)

    # Repeated runs after the timed regions, after the benchmarking method of
    # "Hilbert-Guided Sparse Local Attention": RUNS runs of `iters` launches,
    # the first quarter of each run untimed, each run's mean per launch; the
    # median and minimum over runs go beside the timed region's mean.
    runs_ms = []
    if not args.no_repeats:
        iters = int(min(100, max(8, REPEAT_BUDGET_S * 1e3 / RUNS / max(per_launch_ms, 1e-3))))
        warm = iters // 4
        for _ in range(RUNS):
            for i in range(warm):
                flush_l2(i)
                step()
            r_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                    for _ in range(iters - warm)]
            r0 = torch.cuda.Event(enable_timing=True)
            r1 = torch.cuda.Event(enable_timing=True)
            r0.record(stream)
            for i in range(iters - warm):
                flush_l2(i)
                r_ev[i][0].record(stream)
                step()
                r_ev[i][1].record(stream)
            r1.record(stream)
            torch.cuda.synchronize()
            run_ms = (float(np.sum([a.elapsed_time(b) for a, b in r_ev])) if flush
                      else r0.elapsed_time(r1))
            runs_ms.append(run_ms / (iters - warm))
        na.na_sync_status(stream)
    runs_med = float(np.median(runs_ms)) if runs_ms else per_launch_ms
    runs_min = float(np.min(runs_ms)) if runs_ms else per_launch_ms
    step_med = float(np.median(step_ms))
    step_min = float(np.min(step_ms))

    # Measured speedup over dense attention run through the same kernel (window
    # = the whole grid), after the timed regions: the counterpart of the
    # scheduler's speedup bound (na_plan_info.speedup_bound).
    dense_ms = 0.0
    if not args.no_speedup:
        nd = len(w["grid"])

        def dense_step():
            # full (non-causal) attention, as the scheduler's bound counts it
            na.na_forward(q, k, v, out, lse, w["grid"], [1] * nd, None, stream=stream)

        dense_step()
        d_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(DENSE_STEPS)]
        for i in range(DENSE_STEPS):
            flush_l2(i)
            d_ev[i][0].record(stream)
            dense_step()
            d_ev[i][1].record(stream)
        torch.cuda.synchronize()
        na.na_sync_status(stream)
        dense_ms = float(np.mean([a.elapsed_time(b) for a, b in d_ev]))

    # Context only: the same dense attention through torch's fused
    # scaled_dot_product_attention (a library kernel, never on the measured
    # path), over the flattened token sequence.
    sdpa_ms = 0.0
    if not args.no_speedup and w["dtype"] in ("bf16", "f16"):   # (torch has no E4M3 attention)
        import torch.nn.functional as F
        BH_ = w["B"] * w["heads"]
        N_ = int(np.prod(w["grid"]))
        qs, ks, vs = (t.view(w["B"], w["heads"], N_, w["head_dim"]) for t in (q, k, v))
        try:
            F.scaled_dot_product_attention(qs, ks, vs)
            s_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                    for _ in range(DENSE_STEPS)]
            for i in range(DENSE_STEPS):
                flush_l2(i)
                s_ev[i][0].record(stream)
                F.scaled_dot_product_attention(qs, ks, vs)
                s_ev[i][1].record(stream)
            torch.cuda.synchronize()
            sdpa_ms = float(np.mean([a.elapsed_time(b) for a, b in s_ev]))
        except RuntimeError:
            sdpa_ms = 0.0
        del BH_

    total_ms, e2e_ms, per_launch_ms, dense_ms, sdpa_ms, runs_med, runs_min = max_over_ranks(
        [total_ms, e2e_ms, per_launch_ms, dense_ms, sdpa_ms, runs_med, runs_min], world, dev)

    plan = na.na_plan(w["grid"], w["window"], w["stride"], w["tile"], w["head_dim"],
                      {"bf16": na.NA_BF16, "f16": na.NA_F16, "f32": na.NA_F32,
                       "e4m3": na.NA_E4M3}[w["dtype"]],
                      options=opts)
    flops = flops_per_step(plan["useful_pairs"])
    value = whole_job_tflops(flops, args.steps, world, total_ms)
    e2e_value = whole_job_tflops(flops, args.steps, world, e2e_ms)
    peak, peak_sustained, peak_kind = read_peaks()
    if w["dtype"] == "e4m3":
        # 8-bit products: the measured bf16 rate times the nominal dense
        # fp8 : bf16 ratio (4.5 : 2.25 PFLOP/s)
        peak *= FP8_PER_BF16
    achieved = flops / (per_launch_ms / 1e3) / 1e12
    # The bound: tensor cores when the workload's algorithmic intensity (FLOPs
    # per minimum HBM byte) is above the measured ridge, else HBM bandwidth.
    hbm_peak, hbm_kind = read_hbm_peak()
    min_bytes = min_hbm_bytes()
    hbm_bound = flops / min_bytes < peak * 1e12 / (hbm_peak * 1e9)
    if hbm_bound:
        gbs = min_bytes / (per_launch_ms / 1e3) / 1e9
        roofline = {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
                    "frac": gbs / hbm_peak, "traffic": None,
                    "algorithmic_bytes": min_bytes,
                    "peak_kind": (f"{hbm_kind} copy bandwidth (MEASURED_PEAKS.json)"
                                  if hbm_kind == "measured" else "fallback"),
                    "intensity_flop_per_byte": flops / min_bytes}
    else:
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak,
                    "traffic": read_traffic() if TRAFFIC_APPLIES else None,
                    "peak_kind": (f"{peak_kind} burst bf16 (MEASURED_PEAKS.json)"
                                  + (" x 1: f16 and bf16 share the nominal dense rate"
                                     if w["dtype"] == "f16" else "")
                                  + (" x 2: the nominal dense fp8 : bf16 ratio (4.5 : 2.25 "
                                     "PFLOP/s)" if w["dtype"] == "e4m3" else "")
                                  if peak_kind == "measured" else "fallback")}
    if rank != 0:
        return 0
    base = cpu_baseline(qkv_host) if world == 1 and not args.no_cpu_baseline else None
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w["dtype"],
        "data": "synthetic",
        "config": dict(w, l2=(f"inputs ({h2d / 1e9:.2f} GB) under twice the 126 MB L2: L2 flushed "
                              "by a 256 MB write before each timed step, time = sum of per-step "
                              "events" if flush else
                              f"inputs ({h2d / 1e9:.2f} GB) larger than the 126 MB L2; no flush"),
                       qblock=plan["qblock"], kvchunk=plan["kvchunk"],
                       parallelism=f"replicas x{world}" if world > 1 else "single GPU"),
        "pct_of_peak": 100.0 * value / world / peak,
        "roofline": roofline,
        "cpu_baseline": base,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "schedule": ("pipelined: each step's inputs copied in from pinned host memory "
                             "and its out / lse copied back, on two copy streams with two device "
                             "buffer sets, overlapping the neighbouring steps' compute"
                             if pipelined else
                             "serial: copy in, forward, copy out, one step after another")},
        "speedup": None if args.no_speedup else {
            "bound": plan["speedup_bound"], "measured": dense_ms / per_launch_ms,
            "ideal": plan["dense_pairs"] / plan["useful_pairs"], "dense_ms": dense_ms,
            "kernel_ms": per_launch_ms,
            "vs_torch_sdpa": (sdpa_ms / per_launch_ms) if sdpa_ms > 0 else None,
            "torch_sdpa_dense_ms": sdpa_ms if sdpa_ms > 0 else None,
            "note": "dense = the same kernel with the window set to the whole grid, timed "
                    "after the timed region; bound = dense tile units / computed tile units; "
                    "vs_torch_sdpa = torch scaled_dot_product_attention on the same tensors "
                    "as one dense sequence (context only)"},
        "gpu_launches": args.steps,
        "clocks": clocks,
        "kernel_ms": per_launch_ms,
        "kernel_ms_median": runs_med,
        "kernel_ms_min": runs_min,
        "timing": {
            "protocol": (f"{len(runs_ms)} runs x {iters} launches after the timed region, the "
                         f"first {warm} of each run untimed; per run the mean per launch"
                         if runs_ms else "repeats skipped (--no-repeats): timed region only"),
            "runs_ms": runs_ms,
            "runs_median_ms": runs_med, "runs_min_ms": runs_min,
            "timed_region_steps": {"mean_ms": per_launch_ms, "median_ms": step_med,
                                   "min_ms": step_min, "max_ms": float(np.max(step_ms))},
            "median_tflops": flops / (runs_med / 1e3) / 1e12 * world,
            "best_tflops": flops / (runs_min / 1e3) / 1e12 * world},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (na_backward) instead of the forward")
    ap.add_argument("--no-speedup", action="store_true",
                    help="skip timing dense attention for the measured speedup")
    ap.add_argument("--no-repeats", action="store_true",
                    help="skip the repeated runs (median / min) after the timed region")
    ap.add_argument("--config", type=int, default=4, choices=sorted(WORKLOADS),
                    help="workload: 4 (default) is the 3-D sliding tile one the metric is "
                         "quoted on; 1, 2, 3, 5, 6 are the other parity workloads")
    ap.add_argument("--dtype", choices=["bf16", "f16", "e4m3"], default=None,
                    help="input type of a 16-bit workload (default: the workload's own, bf16); "
                         "e4m3: OFP8 E4M3 q, k, v with bf16 out")
    ap.add_argument("--heads", type=int, default=0,
                    help="profiling only: run the workload with this many heads instead of 24 "
                         "(the JSON line then reports that smaller workload)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.backward and args.dtype == "e4m3":
        ap.error("the backward takes fp32, bf16 or f16 inputs (not e4m3)")
    global WORKLOAD, METRIC, TRAFFIC_APPLIES
    if args.config != 4:
        WORKLOAD = WORKLOADS[args.config]
        METRIC = f"effective TFLOP/s, {WORKLOAD['workload']}"
        TRAFFIC_APPLIES = False
    if args.heads > 0:
        WORKLOAD["heads"] = args.heads
        TRAFFIC_APPLIES = False
    if args.dtype and args.dtype != WORKLOAD["dtype"]:
        if WORKLOAD["dtype"] == "f32":
            ap.error("--dtype applies to the 16-bit workloads only")
        WORKLOAD = dict(WORKLOAD, dtype=args.dtype)
        METRIC = f"effective TFLOP/s, {WORKLOAD['workload']}, {args.dtype} inputs"
        TRAFFIC_APPLIES = False
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.backward:
            return run_backward(args, rank, world, local_rank)
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
