"""The product path stands alone: importing every module of the package loads
nothing from oracle/, and without libcg.so the binding raises instead of falling
back to anything (each check in a fresh interpreter)."""
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(code):
    return subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300)


def test_package_imports_nothing_from_the_oracle():
    r = _run(
        "import sys\n"
        "import quantization_cg_encode_b200\n"
        "from quantization_cg_encode_b200 import cg, controls, synth, train, build\n"
        "bad = sorted(m for m in sys.modules if m == 'oracle' or m.startswith('oracle.'))\n"
        "print(bad)\n"
        "sys.exit(1 if bad else 0)\n")
    assert r.returncode == 0, (r.stdout, r.stderr)


def test_missing_library_raises():
    r = _run(
        "from quantization_cg_encode_b200 import cg\n"
        "cg.LIB_PATH = '/nonexistent/libcg.so'\n"
        "try:\n"
        "    cg.lib()\n"
        "except ImportError as e:\n"
        "    print('raised', e)\n"
        "else:\n"
        "    raise SystemExit('no error')\n")
    assert r.returncode == 0 and "raised" in r.stdout, (r.stdout, r.stderr)
