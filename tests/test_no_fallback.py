"""The product path has no fallback: without the built CUDA library the
binding refuses to load, and no product module reaches the oracle."""
import os
import re
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "paged_kv_cache_464_b200")


def test_binding_fails_loudly_without_the_library(tmp_path):
    # a copy of the package's Python files, without libpa_b200.so
    dst = tmp_path / "paged_kv_cache_464_b200"
    dst.mkdir()
    for f in os.listdir(PKG):
        if f.endswith(".py"):
            shutil.copy(os.path.join(PKG, f), dst / f)
    for mod in ("capi", "block_manager"):
        r = subprocess.run([sys.executable, "-c", f"import paged_kv_cache_464_b200.{mod}"], cwd=tmp_path,
                           capture_output=True, text=True, timeout=300,
                           env={**os.environ, "PYTHONPATH": str(tmp_path)})
        assert r.returncode != 0, f"{mod} imported without the library"
        assert "ImportError" in r.stderr and "not built" in r.stderr, r.stderr[-500:]


def test_product_modules_never_import_the_oracle():
    pattern = re.compile(r"^\s*(import\s+oracle|from\s+oracle\b|from\s+\.\.\s*oracle)", re.M)
    for f in sorted(os.listdir(PKG)):
        if f.endswith(".py"):
            text = open(os.path.join(PKG, f)).read()
            assert not pattern.search(text), f"{f} imports the oracle"
    csrc = os.path.join(PKG, "csrc")
    for f in sorted(os.listdir(csrc)):
        text = open(os.path.join(csrc, f)).read()
        assert "pa_oracle" not in text and "oracle/" not in text, f"csrc/{f} refers to the oracle"
