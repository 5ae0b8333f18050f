"""Host-side check of the forward's work-item order (fwd_schedule.h), no GPU needed.

Compiles tests/host_src/fwd_schedule_check.cpp with the system C++ compiler against the
library's schedule header (the same functions the kernel's roles call) and runs it: for
the fused two-pass order and the one-launch k-pass order (2 to 5 passes, 1 to 48 heads,
lags 1 to 3), every (pass, head, pair) is decoded exactly once and every item of pass
j-1 of a head precedes every item of its pass j.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "sub_quadratic_two_b200", "csrc")


@pytest.mark.skipif(shutil.which("g++") is None, reason="no host C++ compiler")
def test_forward_item_order(tmp_path):
    exe = tmp_path / "fwd_schedule_check"
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-I", CSRC,
                           os.path.join(HERE, "host_src", "fwd_schedule_check.cpp"), "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.startswith("ok"), out.stdout + out.stderr
