"""The product path has no CPU fallback: the binding refuses to import without libda.so, and
nothing in the package reaches the oracle (no GPU needed)."""
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "block_sparse_cluster_b200")


def test_binding_fails_loudly_without_the_library(tmp_path):
    pkg = tmp_path / "block_sparse_cluster_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(PKG, "__init__.py"), pkg / "__init__.py")
    r = subprocess.run([sys.executable, "-c", "import block_sparse_cluster_b200"], cwd=tmp_path,
                       env={**os.environ, "PYTHONPATH": str(tmp_path)}, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "libda.so is not built" in r.stderr


def test_package_sources_never_reach_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h", ".inc")):
                src = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in src and "from oracle" not in src, fn
                assert "oracle/" not in src, fn
