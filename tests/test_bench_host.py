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


def test_round_weight_bytes_of_the_64_layer_round():
    # 64 x (q/k/v 15,360 x 5,120 + o 5,120^2 + gate and up 17,408 x 5,120 + down 5,120 x 17,408)
    # + head 151,936 x 5,120, at 0.5625 bytes per weight (all sizes are whole 32 x 64 units)
    elems = 64 * (4 * 5120 * 5120 + 3 * 17408 * 5120) + 151936 * 5120
    assert bench.round_weight_bytes(64, 5120, 17408, 151936) == elems * 9 // 16 == 13_838_376_960
    # a ragged shape pads to whole units
    assert bench.round_weight_bytes(0, 5120, 17408, 33) == 2 * 80 * 1152


def test_reference_arm_config_equals_the_gpu_arm_config():
    import argparse
    args = argparse.Namespace(width=8, layers=64, round_mode="chain")
    a = bench.round_config(args, 1, bench.round_weight_bytes(64, 5120, 17408, 151936), 257, 257)
    assert a["workload"] == "round_64layers_head_m1to8" and a["weight_bytes_per_round"] == 13_838_376_960
    assert a["gemm_nodes"] == a["graph_nodes"] == 257 and a["parallelism"] == "single GPU"
    assert bench.round_config(args, 4, 1, 257, 257)["parallelism"] == "replicas x4"
