"""The product path has no second implementation: the package never reaches the
oracle, and the binding raises instead of falling back when the CUDA library
cannot be built or loaded. CPU only."""

from __future__ import annotations

import ast
import glob
import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "paged_kv_cache_418_b200")


def _imported_modules(path: str):
    tree = ast.parse(open(path, encoding="utf-8").read(), filename=path)
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            for a in node.names:
                yield a.name
        elif isinstance(node, ast.ImportFrom):
            yield node.module or ""
        elif isinstance(node, ast.Call) and getattr(node.func, "id", "") == "__import__":
            yield "<dynamic>"


def test_package_never_imports_the_oracle():
    files = glob.glob(os.path.join(PKG, "**", "*.py"), recursive=True)
    assert files
    for f in files:
        mods = set(_imported_modules(f))
        assert "<dynamic>" not in mods, f
        assert not any(m == "oracle" or m.startswith("oracle.") for m in mods), f
        assert "importlib" not in mods, f


def test_cuda_sources_include_nothing_from_the_oracle():
    for f in glob.glob(os.path.join(PKG, "csrc", "*")) + glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(f, encoding="utf-8").read()
        for inc in re.findall(r'#include\s*[<"]([^>"]+)[>"]', text):
            assert "oracle" not in inc, (f, inc)


def _run(code: str):
    env = dict(os.environ, PYTHONPATH=ROOT)
    return subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env,
                          cwd=ROOT, timeout=300)


def test_binding_raises_when_the_library_cannot_be_built():
    r = _run(
        "import paged_kv_cache_418_b200._build as b\n"
        "def fail():\n"
        "    raise RuntimeError('nvcc not found: the CUDA library cannot be built')\n"
        "b.ensure_built = fail\n"
        "try:\n"
        "    import paged_kv_cache_418_b200.ops\n"
        "except RuntimeError as e:\n"
        "    print('RAISED', e)\n"
        "else:\n"
        "    print('IMPORTED')\n")
    assert r.returncode == 0, r.stderr
    assert "RAISED nvcc not found" in r.stdout, r.stdout


def test_binding_raises_when_the_library_does_not_load(tmp_path):
    bogus = tmp_path / "libpa.so"
    bogus.write_bytes(b"not a shared object")
    r = _run(
        "import paged_kv_cache_418_b200._build as b\n"
        f"b.ensure_built = lambda: {str(bogus)!r}\n"
        "try:\n"
        "    import paged_kv_cache_418_b200.ops\n"
        "except OSError as e:\n"
        "    print('RAISED')\n"
        "else:\n"
        "    print('IMPORTED')\n")
    assert r.returncode == 0, r.stderr
    assert "RAISED" in r.stdout, r.stdout
