"""The product path and the oracle are independent: the package imports and loads its
library with the oracle made unimportable, no package source names the oracle in an import,
and the oracle imports nothing from the package."""

import ast
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "exact_tiled_attention_33_b200")


def _imports(path):
    tree = ast.parse(open(path, encoding="utf-8").read())
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            names.add(node.module.split(".")[0])
    return names


def _py_files(d):
    for base, _, files in os.walk(d):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(base, f)


def test_package_sources_do_not_import_the_oracle():
    for f in _py_files(PKG):
        assert "oracle" not in _imports(f), f


def test_oracle_does_not_import_the_package():
    for f in _py_files(os.path.join(ROOT, "oracle")):
        assert "exact_tiled_attention_33_b200" not in _imports(f), f


def test_package_loads_with_the_oracle_blocked():
    code = ("import sys; sys.modules['oracle'] = None\n"
            "import exact_tiled_attention_33_b200 as p\n"
            "from exact_tiled_attention_33_b200 import _lib, attention, workloads\n"
            "lib = _lib.load()\n"
            "assert lib.fa_bwd_workspace_size(1, 128, 1, 64) == 512 + 128 * 64 * 4\n"
            "assert 'oracle' not in [m for m in sys.modules if sys.modules[m] is not None]\n"
            "print('isolated ok')\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "isolated ok" in r.stdout
