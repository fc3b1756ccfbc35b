"""Host check of the fused decode kernel's tile dealing.

The dealing (expert_ffn_execution_b200/csrc/deal.h) is plain integer
arithmetic that the kernel compiles for the device; here the same header is
compiled for the host with g++ and checked exhaustively over grid sizes,
active-expert counts and shapes: every down tile goes to exactly one CTA
slot, the cut points are monotone, and the tile-table capacity holds."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_fused_dealing_is_a_bijection_within_capacity(tmp_path):
    exe = tmp_path / "deal_check"
    src = os.path.join(ROOT, "tests", "native", "deal_check.cpp")
    inc = os.path.join(ROOT, "expert_ffn_execution_b200", "csrc")
    subprocess.run(["g++", "-std=c++17", "-O2", "-I", inc, src, "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok "), r.stdout
