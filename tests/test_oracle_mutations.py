"""The oracle's pins bite: each plausible mistake below, planted in a copy of
the oracle's C source (in a scratch directory, never in the oracle itself),
makes the pin files fail.  Mistakes covered: swapped nibble order, a reversed
scale index, a dropped E2M1 or E4M3 sign, a wrong E4M3 subnormal exponent,
a dropped global scale, the wrong sign inside SiLU, reversed top-k tie order,
and the wrong order among negative NaNs."""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_FILES = ["tests/test_oracle.py", "tests/test_oracle_topk.py", "tests/test_oracle_properties.py"]

MUTATIONS = {
    "nibble_order": ("return (k & 1) ? (byte >> 4) : (byte & 15u);",
                     "return (k & 1) ? (byte & 15u) : (byte >> 4);"),
    "scale_index": ("return s[n * (K / 16) + k / 16];",
                    "return s[n * (K / 16) + (K / 16 - 1 - k / 16)];"),
    "e4m3_sign_dropped": ("unsigned s = (b >> 7) & 1u,", "unsigned s = 0u * ((b >> 7) & 1u),"),
    "e2m1_sign_dropped": ("unsigned s = (c >> 3) & 1u,", "unsigned s = 0u * ((c >> 3) & 1u),"),
    "e4m3_subnormal_exponent": ("if (e == 0) mag = ldexp((double)m / 8.0, -6);",
                                "if (e == 0) mag = ldexp((double)m / 8.0, -7);"),
    "gscale_dropped": ("            Y[(int64_t)m * N + n] = (double)gscale * acc;",
                       "            Y[(int64_t)m * N + n] = acc;"),
    "silu_sign": ("H[i] = g / (1.0 + exp(-g)) * U[i];", "H[i] = g / (1.0 + exp(g)) * U[i];"),
    "topk_tie_order": ("return (x->i < y->i) ? -1 : (x->i > y->i ? 1 : 0);",
                       "return (x->i < y->i) ? 1 : (x->i > y->i ? -1 : 0);"),
    "topk_negative_nan_order": ("    return px > py ? 1 : -1;", "    return px > py ? -1 : 1;"),
}


def _copy_tree(dst):
    keep = shutil.ignore_patterns("_build", "__pycache__", "*.so", ".pytest_cache", ".hypothesis")
    for d in ("oracle", "tests", "nvfp4_weight_streaming_decode_b200"):
        shutil.copytree(os.path.join(ROOT, d), os.path.join(dst, d), ignore=keep)


def test_unmutated_copy_passes(tmp_path):
    _copy_tree(str(tmp_path))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PIN_FILES],
                       cwd=str(tmp_path), capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_the_pins(tmp_path, name):
    before, after = MUTATIONS[name]
    _copy_tree(str(tmp_path))
    path = os.path.join(str(tmp_path), "oracle", "nvfp4_oracle.c")
    with open(path) as f:
        src = f.read()
    assert src.count(before) == 1, f"mutation site of {name} not found once"
    with open(path, "w") as f:
        f.write(src.replace(before, after))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PIN_FILES],
                       cwd=str(tmp_path), capture_output=True, text=True, timeout=600)
    assert r.returncode == 1, f"{name}: the pins did not catch it\n" + r.stdout[-2000:] + r.stderr[-2000:]
