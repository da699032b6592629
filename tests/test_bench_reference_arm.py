"""bench.py's reference arm (the fp64 oracle timed on the host cores), run on
CPU at the smallest workload: one JSON line with the contract's keys, a sample
that never exceeds the workload's own query rows, and, under a two-process
launch, a line from rank 0 only while the other rank exits 0 without work."""
import json
import os
import socket
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402

KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
        "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
        "cpu_baseline", "e2e"}


def _json_lines(text):
    return [json.loads(l) for l in text.splitlines() if l.startswith("{")]


def test_sample_rows_never_exceed_the_workload(monkeypatch):
    monkeypatch.setattr(bench, "WORKLOAD", dict(bench.WORKLOAD, B=1, heads=2, grid=[16, 16]))
    assert bench.workload_rows() == 512
    rows = bench.oracle_sample_rows(10_000)
    assert np.array_equal(rows, np.arange(512))
    rows = bench.oracle_sample_rows(100)
    assert len(rows) == 100 and len(np.unique(rows)) == 100
    assert rows.min() >= 0 and rows.max() < 512 and np.all(np.diff(rows) > 0)


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "1",
                          "--steps", "1", "--warmup", "3"],
                         cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = _json_lines(out.stdout)
    assert len(lines) == 1
    line = lines[0]
    assert KEYS <= set(line)
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    # the 16 x 16 grid with 2 heads has 512 query rows: the whole workload is the sample
    assert line["config"]["sample_rows_per_step"] == 512


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_reference_arm_two_ranks_only_rank0_prints():
    env = dict(os.environ, MASTER_ADDR="127.0.0.1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl",
           "reference", "--gpus", "2", "--config", "1", "--steps", "1", "--warmup", "3"]
    out = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = _json_lines(out.stdout)
    assert len(lines) == 1
    assert lines[0]["impl"] == "reference" and lines[0]["n_gpus"] == 2
