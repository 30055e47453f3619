"""The product path stands alone: without its CUDA library it raises instead
of computing anything another way, and importing it never loads the oracle
(which is test infrastructure only).  Each check runs in a fresh interpreter."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(code, **env):
    e = dict(os.environ, PYTHONPATH=ROOT, **env)
    return subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT, env=e,
                          timeout=300)


def test_missing_library_raises_on_load_and_on_every_call():
    code = (
        "from nvfp4_weight_streaming_decode_b200 import abi\n"
        "for f in (abi.load, lambda: abi.nvfp4_version(), lambda: abi.nvfp4_packed_bytes(32, 64)):\n"
        "    try:\n"
        "        f()\n"
        "    except RuntimeError as e:\n"
        "        assert 'missing' in str(e), e\n"
        "    else:\n"
        "        raise SystemExit('no error without the library')\n"
        "print('raised')\n")
    r = _run(code, NVFP4_LIB=os.path.join(ROOT, "no_such_dir", "libnvfp4decode.so"))
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "raised"


def test_product_modules_do_not_import_the_oracle():
    code = (
        "import sys\n"
        "import nvfp4_weight_streaming_decode_b200\n"
        "from nvfp4_weight_streaming_decode_b200 import abi, build, synth, workloads\n"
        "abi.load()\n"
        "bad = [m for m in sys.modules if m == 'oracle' or m.startswith('oracle.')]\n"
        "assert not bad, bad\n"
        "print('clean')\n")
    r = _run(code)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "clean"


def test_product_sources_name_no_oracle():
    pkg = os.path.join(ROOT, "nvfp4_weight_streaming_decode_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                with open(os.path.join(dirpath, f)) as fh:
                    text = fh.read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "nvfp4_oracle" not in text and "liboracle" not in text, f
