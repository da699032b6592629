"""The tensor-core kernels' chunk walks, compiled for the host with g++ from
the CUDA path's host/device scheduler headers and checked by brute force on
random 1-D, 2-D and 3-D problems in every window mode: the forward's walk
over key chunks for a CTA's two query blocks, and the dK / dV kernel's walk
over query chunks for one key block.  Each visits every chunk that holds an
attended pair, only such chunks, and marks FULL (no mask) only chunks inside
the grid where every pair is attended."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "neighborhood_attention_b200", "csrc")


def _run(tmp_path, name):
    exe = tmp_path / name
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-I", CSRC, "-o", str(exe),
                           os.path.join(ROOT, "tests", name + ".cpp")])
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert " 0 wrong" in out.stdout, out.stdout


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_forward_cta_pair_walk(tmp_path):
    _run(tmp_path, "cta_pair_walk_check")


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_backward_key_block_walk(tmp_path):
    _run(tmp_path, "key_block_walk_check")
