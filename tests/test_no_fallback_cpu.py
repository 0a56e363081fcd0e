"""The product path has no fallback (CPU only).

- Importing the package without its compiled library raises ImportError
  instead of quietly running something else.
- No module of the package, nor bench.py's timed path, imports the float64
  oracle: the oracle is test infrastructure, used only by the tests, by the
  smoke check, and by the benchmark's CPU-baseline and reference legs.
"""
import ast
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "sliding_window_attention_tc_b200")


def test_import_without_library_fails_loudly(tmp_path):
    dst = tmp_path / "sliding_window_attention_tc_b200"
    dst.mkdir()
    for f in os.listdir(PKG):
        if f.endswith(".py"):
            shutil.copy(os.path.join(PKG, f), dst / f)
    assert not (dst / "libtc.so").exists()
    r = subprocess.run([sys.executable, "-c", "import sliding_window_attention_tc_b200"],
                       cwd=tmp_path, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "libtc.so" in r.stderr


def _imported_modules(path):
    tree = ast.parse(open(path).read())
    mods = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            mods.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module:
            mods.add(node.module.split(".")[0])
    return mods


def test_package_never_imports_the_oracle():
    for f in os.listdir(PKG):
        if f.endswith(".py"):
            assert "oracle" not in _imported_modules(os.path.join(PKG, f)), f


def test_bench_imports_the_oracle_only_in_its_cpu_legs():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    assert "oracle" not in {a.name.split(".")[0] for n in tree.body if isinstance(n, ast.Import)
                            for a in n.names}
    users = set()
    for fn in ast.walk(tree):
        if isinstance(fn, ast.FunctionDef):
            for node in ast.walk(fn):
                if isinstance(node, ast.Import) and any(a.name.split(".")[0] == "oracle"
                                                        for a in node.names):
                    users.add(fn.name)
                if isinstance(node, ast.ImportFrom) and (node.module or "").startswith("oracle"):
                    users.add(fn.name)
    assert users, "bench.py is expected to time the oracle for its CPU baseline"
    for name in users:
        assert "oracle" in name or "reference" in name or "cpu" in name, name
