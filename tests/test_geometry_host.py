"""Host-side check of the CUDA path's index arithmetic (geometry.h), no GPU needed.

Compiles tests/host_src/geometry_check.cpp with the system C++ compiler against the
library's geometry header and runs it: the multiply-shift division (FastDiv) must
equal integer division for every divisor up to 4096 and for random 31-bit operands,
and the problem, tile and row offsets must equal their plain-division definitions
over random nested tilings.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "sub_quadratic_two_b200", "csrc")


@pytest.mark.skipif(shutil.which("g++") is None, reason="no host C++ compiler")
def test_geometry_index_arithmetic(tmp_path):
    exe = tmp_path / "geometry_check"
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-I", CSRC, os.path.join(HERE, "host_src", "geometry_check.cpp"),
                           "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.startswith("ok"), out.stdout + out.stderr
