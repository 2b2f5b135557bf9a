"""The product path has no fallback: importing the package without the CUDA
library fails, and the package never imports the oracle."""
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = "exact_io_aware_55_b200"


def test_import_without_library_fails_loudly(tmp_path):
    dst = tmp_path / PKG
    shutil.copytree(os.path.join(ROOT, PKG), dst,
                    ignore=shutil.ignore_patterns("*.so", "*.sha256", "__pycache__", "csrc"))
    assert not (dst / "libfa.so").exists()
    r = subprocess.run([sys.executable, "-c", f"import {PKG}"], cwd=tmp_path, capture_output=True, text=True)
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "no CPU fallback" in r.stderr


def test_package_does_not_import_the_oracle():
    code = (f"import sys; sys.path.insert(0, {ROOT!r}); import {PKG}; "
            "assert 'oracle' not in sys.modules, 'product path imported the oracle'; print('ok')")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"
