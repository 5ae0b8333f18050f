"""Host-side checks of bench.py helpers that tie committed ncu counters to kernel sources."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_only_drops_comments_and_blank_lines():
    src = "int a = 1;  // one\n\n/* block\n comment */int b = 2;\n   // only a comment\nint c; /* x */ int d;\n"
    assert bench.code_only(src) == "int a = 1;\nint b = 2;\nint c;  int d;"


def test_source_sha_ignores_comments_but_not_code(tmp_path):
    a, b, c = tmp_path / "a.cuh", tmp_path / "b.cuh", tmp_path / "c.cuh"
    a.write_text("__device__ int f(int x) { return x + 1; }  // add one\n")
    b.write_text("// a different comment\n__device__ int f(int x) { return x + 1; }\n\n")
    c.write_text("__device__ int f(int x) { return x + 2; }\n")
    assert bench.source_sha([str(a)]) == bench.source_sha([str(b)])
    assert bench.source_sha([str(a)]) != bench.source_sha([str(c)])


def test_read_traffic_needs_a_matching_hash(tmp_path):
    other = tmp_path / "k.cuh"
    other.write_text("__global__ void k() {}\n")
    assert bench.read_traffic("fused", [str(other)]) is None
