"""Host check of the per-device, per-context address cache that the
allocation-free decode entry point uses for its in-library scratch array:
compiled with g++ against fake contexts and a fake symbol lookup."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_address_cache_is_keyed_by_device_and_context(tmp_path):
    exe = tmp_path / "scratch_cache_check"
    src = os.path.join(ROOT, "tests", "native", "scratch_cache_check.cpp")
    inc = os.path.join(ROOT, "expert_ffn_execution_b200", "csrc")
    subprocess.run(["g++", "-std=c++17", "-O1", "-pthread", "-I", inc, src, "-o", str(exe)],
                   check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok "), r.stdout
