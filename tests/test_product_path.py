"""The product path never reaches the oracle and has no CPU fallback.

* No module of the package imports or names the oracle.
* bench.py imports the oracle only inside its CPU-baseline helper, and
  __graft_entry__ only inside build() (which compiles it) and smoke() (which
  checks against it).
* libmoefp8.so neither links liboracle nor carries an oracle symbol.
* Importing the package without the built library raises ImportError.
"""
import ast
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "sparse_moe_layer_expert_b200")


def _oracle_imports(path):
    """(enclosing function or '<module>', line) of every import of the oracle."""
    tree = ast.parse(open(path).read(), path)
    found = []

    def visit(node, func):
        for child in ast.iter_child_nodes(node):
            f = child.name if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)) else func
            if isinstance(child, ast.Import) and any(a.name.split(".")[0] == "oracle" for a in child.names):
                found.append((func, child.lineno))
            elif isinstance(child, ast.ImportFrom) and (child.module or "").split(".")[0] == "oracle":
                found.append((func, child.lineno))
            visit(child, f)

    visit(tree, "<module>")
    return found


def test_package_never_imports_or_names_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if not f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                continue
            p = os.path.join(dirpath, f)
            if f.endswith(".py"):
                assert not _oracle_imports(p), p
            src = open(p).read()
            assert "liboracle" not in src and "moe_oracle" not in src, p


def test_bench_and_entry_points_import_the_oracle_only_where_allowed():
    bench = _oracle_imports(os.path.join(ROOT, "bench.py"))
    assert bench and {fn for fn, _ in bench} == {"oracle_sample"}, bench
    entry = _oracle_imports(os.path.join(ROOT, "__graft_entry__.py"))
    assert entry and {fn for fn, _ in entry} <= {"build", "smoke"}, entry


@pytest.mark.skipif(shutil.which("readelf") is None or shutil.which("nm") is None, reason="binutils not found")
def test_library_does_not_link_or_contain_the_oracle():
    lib = os.path.join(PKG, "libmoefp8.so")
    if not os.path.exists(lib):
        pytest.skip("library not built")
    needed = subprocess.run(["readelf", "-d", lib], capture_output=True, text=True, check=True).stdout
    assert "oracle" not in needed
    syms = subprocess.run(["nm", "-D", lib], capture_output=True, text=True, check=True).stdout
    assert "moe_oracle" not in syms


def test_import_without_the_library_fails_loudly(tmp_path):
    dst = tmp_path / "sparse_moe_layer_expert_b200"
    dst.mkdir()
    for f in os.listdir(PKG):
        if f.endswith(".py"):
            shutil.copy(os.path.join(PKG, f), dst / f)
    r = subprocess.run([sys.executable, "-c", "import sparse_moe_layer_expert_b200"], cwd=tmp_path,
                       env=dict(os.environ, PYTHONPATH=str(tmp_path)), capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "libmoefp8.so is missing" in r.stderr
