"""Host-side arithmetic of bench.py, on CPU: the FLOP count per step, the
algorithmic HBM bytes behind the HBM roofline, the rule that a stored ncu
traffic figure applies only to the kernel sources it was taken on, and the
peak fallbacks."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_flops_count_four_d_per_attended_pair():
    w = bench.WORKLOADS[4]        # 3-D sliding tile: every query sees 18*24*40 keys
    pairs = 30 * 48 * 80 * 18 * 24 * 40
    assert bench.flops_per_step(pairs, w) == 4.0 * 128 * 1 * 24 * pairs
    # two matrix products (Q K^T and P V) of 2 d FLOPs per pair each
    assert bench.flops_per_step(1, dict(w, B=1, heads=1)) == 2 * (2 * 128)


def test_min_hbm_bytes_of_the_long_1d_workload():
    w = bench.WORKLOADS[6]        # 16 heads x 32768 tokens, d 64, bf16
    tokens = 16 * 32768
    # q, k, v read and out written (d bf16 values each), lse written (fp32)
    assert bench.min_hbm_bytes(w) == tokens * (4 * 64 * 2 + 4)
    assert bench.min_hbm_bytes(w) == 270_532_608
    f32 = dict(w, dtype="f32")
    assert bench.min_hbm_bytes(f32) == tokens * (4 * 64 * 4 + 4)


def test_hbm_workload_sits_below_the_ridge_and_sta_above():
    # FLOPs per algorithmic byte against the fallback ridge (both peaks from
    # the same pool): the 1-D causal w = 5 workload is far below it, the 3-D
    # sliding tile workload far above.
    ridge = bench.FALLBACK_PEAK_TFLOPS * 1e12 / (bench.FALLBACK_HBM_GBS * 1e9)
    w6 = bench.WORKLOADS[6]
    i6 = bench.flops_per_step(32768 * 5, w6) / bench.min_hbm_bytes(w6)
    w4 = bench.WORKLOADS[4]
    i4 = bench.flops_per_step(30 * 48 * 80 * 18 * 24 * 40, w4) / bench.min_hbm_bytes(w4)
    assert i6 < 5 < ridge < 1000 < i4


def test_traffic_figure_applies_only_to_its_sources(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("// kernel v1\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", ["kernel.cu"])
    tf = tmp_path / "traffic.txt"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tf))
    tf.write_text(f"# comment\nkernel_hash {bench.kernel_hash()}\ndram_bytes_per_launch 12345\n")
    assert bench.read_traffic() == 12345.0
    src.write_text("// kernel v2\n")             # the kernel changed since the capture
    assert bench.read_traffic() is None
    tf.write_text("kernel_hash 0\n")             # malformed / missing figure
    assert bench.read_traffic() is None


def test_peaks_fall_back_without_measured_file(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.read_peaks() == (bench.FALLBACK_PEAK_TFLOPS, 0.0, "fallback")
    assert bench.read_hbm_peak() == (bench.FALLBACK_HBM_GBS, "fallback")
    (tmp_path / "MEASURED_PEAKS.json").write_text(
        json.dumps({"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6500.0}))
    assert bench.read_peaks() == (1600.0, 1400.0, "measured")
    assert bench.read_hbm_peak() == (6500.0, "measured")


def test_whole_job_value_counts_every_rank():
    # 3 steps of 2e12 FLOPs on each of 4 ranks in 10 ms (slowest rank)
    assert bench.whole_job_tflops(2e12, 3, 4, 10.0) == pytest.approx(2400.0)
