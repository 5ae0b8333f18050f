"""Host check of the tensor-map cache (csrc/tmap_cache.h), no GPU needed.

Compiles tests/host_src/tmap_cache_check.cpp against the cache header and the CUDA
driver header (types only, nothing is linked or called) and runs it: a repeated
call with the same pointers and shapes performs no encode and gets the map made for
it; any other pointer, shape, box or device is encoded; the least recently used
entry is evicted; failures are not cached; eight threads hammering the cache get the
right map for every key.
"""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "sub_quadratic_two_b200", "csrc")


def _cuda_include():
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.realpath(nvcc))), "include")
    return inc if os.path.exists(os.path.join(inc, "cuda.h")) else None


@pytest.mark.skipif(shutil.which("g++") is None or _cuda_include() is None, reason="no host C++ compiler or cuda.h")
def test_tensor_map_cache(tmp_path):
    exe = tmp_path / "tmap_cache_check"
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-pthread", "-I", CSRC, "-I", _cuda_include(),
                           os.path.join(HERE, "host_src", "tmap_cache_check.cpp"), "-o", str(exe)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and out.stdout.startswith("ok"), out.stdout + out.stderr
