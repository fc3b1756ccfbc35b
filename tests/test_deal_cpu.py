"""Host checks of the fused decode kernel's tile dealing and synchronisation.

The dealing (expert_ffn_execution_b200/csrc/deal.h) is plain integer
arithmetic that the kernel compiles for the device; here the same header is
compiled for the host with g++ and checked exhaustively over grid sizes,
active-expert counts and shapes: every down tile goes to exactly one CTA
slot, the cut points are monotone, and the tile-table capacity holds.

The synchronisation check runs a model of the fused kernel's barrier
protocol (tests/native/pipeline_check.cpp) over the same dealing under
random interleavings: it completes exactly when the in-flight capacity
condition holds, deadlocks otherwise, and flags a parity hazard for four
decoder groups on three tensor-memory stages."""
import os
import re
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


def _kernel_source():
    with open(os.path.join(ROOT, "expert_ffn_execution_b200", "csrc",
                           "experts_decode_tc.cu")) as f:
        return f.read()


def test_pipeline_model_uses_the_kernels_counts():
    """The model runs three decoder groups, one tensor-memory stage per
    group, 256-K chunks and stage counts that are multiples of three up to
    15; the kernel's constants and its fused-form condition must match."""
    src = _kernel_source()
    const = dict(re.findall(r"constexpr int (kTc\w+) = (\d+);", src))
    assert const["kTcGroups"] == "3" and const["kTcTS"] == "3"
    assert const["kTcKC"] == "256" and const["kTcMaxStages"] == "16"
    assert "S + 2 * kTcGroups >= nchB" in src


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_fused_pipeline_model_completes_exactly_within_capacity(tmp_path):
    exe = tmp_path / "pipeline_check"
    src = os.path.join(ROOT, "tests", "native", "pipeline_check.cpp")
    inc = os.path.join(ROOT, "expert_ffn_execution_b200", "csrc")
    subprocess.run(["g++", "-std=c++17", "-O2", "-I", inc, src, "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.splitlines()[-1].startswith("ok "), r.stdout
    assert "flagged as expected" in r.stdout
