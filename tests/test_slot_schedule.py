"""The backward pipelines' stage slots (the CUDA path's host/device header,
compiled for the host with g++): the two tiles of a chunk share its stage,
the roles swap every round, and each slot's fill number is the chunk's
round, as the barrier parities of the producer and the MMA issuer assume."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_stage_slots_swap_roles_and_fill_once_per_round(tmp_path):
    exe = tmp_path / "slot_schedule_check"
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-I",
                           os.path.join(ROOT, "neighborhood_attention_b200", "csrc"),
                           "-o", str(exe), os.path.join(ROOT, "tests", "slot_schedule_check.cpp")])
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert " 0 wrong" in out.stdout
