"""The key mask of partial chunks (the CUDA path's host/device header,
compiled for the host with g++) agrees bit for bit with a direct per-key
window test over every 128-key chunk shape."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_chunk_key_mask_matches_per_key_test(tmp_path):
    exe = tmp_path / "chunk_mask_check"
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-I",
                           os.path.join(ROOT, "neighborhood_attention_b200", "csrc"),
                           "-o", str(exe), os.path.join(ROOT, "tests", "chunk_mask_check.cpp")])
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert " 0 wrong" in out.stdout
