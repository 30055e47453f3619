"""Host-side helpers of bench.py (no GPU): the kernel-source hash that ties the
committed DRAM-traffic summary to the decode GEMM's code ignores comments and
blank lines, and nothing else."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402


def test_kernel_code_drops_comments_and_blank_lines():
    src = "int a; // note\n\n/* block\n comment */ int b;\n   \nint c; /* x */ int d;\n"
    assert bench.kernel_code(src) == "int a;\n int b;\nint c;  int d;"


def test_kernel_code_keeps_code_changes_visible():
    a = "x = y + 1; // one\n"
    b = "x = y + 2; // one\n"
    assert bench.kernel_code(a) != bench.kernel_code(b)
    assert bench.kernel_code(a) == bench.kernel_code("x = y + 1; // another comment\n")


def test_kernel_hash_is_stable():
    h = bench.kernel_hash()
    assert len(h) == 16 and h == bench.kernel_hash()
