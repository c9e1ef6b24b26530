"""The oracle and the CUDA path share no code: the product package never
imports or loads the oracle, the oracle never includes or imports the
product's sources, and the product fails loudly (ImportError) when its
library is missing instead of falling back to anything."""
import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "precision_weight_quantization_b200")
ORACLE = os.path.join(ROOT, "oracle")


def files(d, exts):
    for base, _, names in os.walk(d):
        for n in names:
            if n.endswith(exts):
                yield os.path.join(base, n)


def test_product_never_touches_the_oracle():
    for f in files(PKG, (".py", ".cu", ".cuh", ".h", ".cpp")):
        text = open(f, encoding="utf-8").read()
        assert not re.search(r"^\s*(from|import)\s+oracle\b", text, re.M), f
        assert "pwq_oracle" not in text and "libpwq_oracle" not in text, f


def test_oracle_never_touches_the_product():
    for f in files(ORACLE, (".py", ".c", ".h")):
        text = open(f, encoding="utf-8").read()
        assert "precision_weight_quantization_b200" not in text, f
        assert "pwq_device" not in text and "libpwq.so" not in text and "pwq.h" not in text, f


def test_workloads_hold_no_quantisation_arithmetic():
    text = open(os.path.join(ROOT, "workloads.py"), encoding="utf-8").read()
    assert not re.search(r"^\s*(from|import)\s+(oracle|precision_weight_quantization_b200)\b", text, re.M)
    for word in ("448", "2688", "e4m3", "e2m1", "ue8m0"):
        assert word not in text.lower(), word


def test_missing_library_fails_loudly(tmp_path):
    # a copy of the package without libpwq.so must refuse to import
    import shutil
    dst = tmp_path / "precision_weight_quantization_b200"
    shutil.copytree(PKG, dst, ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    code = ("import sys; sys.path.insert(0, %r)\n"
            "try:\n    import precision_weight_quantization_b200\nexcept ImportError as e:\n"
            "    print('ImportError', e); sys.exit(0)\nsys.exit(1)\n" % str(tmp_path))
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0 and "libpwq.so is not built" in out.stdout, out.stdout + out.stderr
