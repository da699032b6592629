"""The key-stationary dK / dV kernel's inverse windows (the CUDA path's
host/device header, compiled for the host with g++): for every key, exactly
the queries whose window holds it, as an interval that moves monotonically
with the key, in every window mode; and for every key block, the query box
the kernel takes from its first and last keys (queries that see some key of
the block) and the box's core (queries that see all of them)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_inverse_range_is_the_set_of_queries_that_see_the_key(tmp_path):
    exe = tmp_path / "inverse_window_check"
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-I",
                           os.path.join(ROOT, "neighborhood_attention_b200", "csrc"),
                           "-o", str(exe), os.path.join(ROOT, "tests", "inverse_window_check.cpp")])
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.count(" 0 wrong") == 2, out.stdout

