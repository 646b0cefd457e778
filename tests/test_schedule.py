"""Host logic: the GEMM tile schedules cover every output tile exactly once.

Compiles tests/native/schedule_check.cpp (which includes the schedule header
the kernels use) with g++ and runs it; no GPU needed."""

import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_tile_schedules_cover_each_tile_once(tmp_path):
    exe = tmp_path / "schedule_check"
    subprocess.run(["g++", "-std=c++17", "-O2", "-o", str(exe),
                    os.path.join(HERE, "native", "schedule_check.cpp")], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert out.returncode == 0 and out.stdout.startswith("OK"), out.stdout + out.stderr
