"""Host-side helpers of bench.py (no GPU): the kernel-source hash that ties the
committed DRAM-traffic summary to the decode GEMM's code ignores comments and
blank lines, and nothing else; the percentile used for the per-replay round
times agrees with numpy's."""
import os
import sys

import pytest

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


@pytest.mark.parametrize("xs", [[1.0], [2.0, 1.0], [float(i) for i in range(20)], [0.3, 5.1, 4.9, 5.0, 7.2, 5.05]])
@pytest.mark.parametrize("q", [0, 50, 90, 100])
def test_percentile_matches_numpy(xs, q):
    import numpy as np
    assert bench.percentile(xs, q) == pytest.approx(float(np.percentile(xs, q)), rel=1e-12, abs=1e-12)
