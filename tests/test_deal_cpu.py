"""Host checks of the fused decode kernel's tile dealing and synchronisation.

The dealing (expert_ffn_execution_b200/csrc/deal.h) is plain integer
arithmetic that the kernel compiles for the device; here the same header is
compiled for the host with g++ and checked exhaustively over grid sizes,
active-expert counts and shapes: every down tile goes to exactly one CTA
slot, the cut points are monotone, and the tile-table capacity holds.

The synchronisation check runs models of the expert kernels' barrier
protocols (tests/native/pipeline_check.cpp) under random interleavings: the
fused decode kernel over the same dealing completes exactly when the
in-flight capacity condition holds, deadlocks otherwise, and shows a parity
hazard for four decoder groups on three tensor-memory stages; both grids of
the two-kernel decode form complete for every stage count; the prefill
grouped GEMM completes for both code widths over K sizes and unit counts.
Abort runs (an abort raised at a random step, then the kernels' drains)
stay clean when a role releases no buffer after any of its waits gave up;
with the releases as the kernels make them, some abort run starts a copy
into a buffer whose previous copy is still landing."""
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


def _prefill_source():
    with open(os.path.join(ROOT, "expert_ffn_execution_b200", "csrc",
                           "experts_prefill.cu")) as f:
        return f.read()


def test_pipeline_model_uses_the_kernels_counts():
    """The decode model runs three decoder groups, one tensor-memory stage
    per group, 256-K chunks and stage counts that are multiples of three up
    to 15; the prefill model four A/B stages, three code stages of 64 code
    bytes per row (4 chunks of 2-bit codes, 2 of 4-bit), two producer groups
    each releasing a code stage after its last chunk in it.  The kernels'
    constants and conditions must match."""
    src = _kernel_source()
    const = dict(re.findall(r"constexpr int (kTc\w+) = (\d+);", src))
    assert const["kTcGroups"] == "3" and const["kTcTS"] == "3"
    assert const["kTcKC"] == "256" and const["kTcMaxStages"] == "16"
    assert "S + 2 * kTcGroups >= nchB" in src
    pre = _prefill_source()
    assert "static constexpr int S = 4;" in pre and "static constexpr int CSN = 3;" in pre
    assert "constexpr int kPCodeRow = 64;" in pre and "constexpr int kPK = 64;" in pre
    assert "return FMT == STRATA_FMT_Q2_32 ? 16 : 32;" in pre
    assert "mbar_init(&cempty[c], 256);" in pre and "mbar_init(&full[s], 128);" in pre
    assert "if (slot + 2 >= in_cs) mbar_arrive(&cempty[ci]);" in pre


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_pipeline_models_complete_exactly_within_capacity(tmp_path):
    exe = tmp_path / "pipeline_check"
    src = os.path.join(ROOT, "tests", "native", "pipeline_check.cpp")
    inc = os.path.join(ROOT, "expert_ffn_execution_b200", "csrc")
    subprocess.run(["g++", "-std=c++17", "-O2", "-I", inc, src, "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.splitlines()[-1].startswith("ok "), r.stdout
    assert "flagged as expected" in r.stdout
    assert "unguarded releases after an abort" in r.stdout
