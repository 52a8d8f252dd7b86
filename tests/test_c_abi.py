"""The C ABI used from C: `tests/c/abi_from_c.c` is compiled as strict C99 against
`include/fattn.h` alone, linked against the in-tree libfattn.so and run.  It calls only
what needs no GPU (workspace sizes, status strings, host-side validation)."""

import os
import shutil
import subprocess

import pytest

from exact_tiled_attention_33_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_header_compiles_as_c99_and_links(tmp_path):
    lib_path = _lib.load()._name
    lib_dir = os.path.dirname(os.path.abspath(lib_path))
    exe = tmp_path / "abi_from_c"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_from_c.c"),
           "-o", str(exe), lib_path, f"-Wl,-rpath,{lib_dir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "all checks passed" in r.stdout
