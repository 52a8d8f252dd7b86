"""CPU check that the Python binding's ctypes signatures match the C header parameter by
parameter: a binding that passed one argument too few, or an int where the C side reads a
float or a 64-bit size, would hand the kernels wrong sizes or pointers without any error.
The header is parsed as text (comments removed); each C parameter type maps to the one
ctypes type that has its size and calling convention."""

import ctypes
import os
import re

from exact_tiled_attention_33_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fattn.h")


def _declarations():
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    decls = {}
    for m in re.finditer(r"([A-Za-z_][\w\s\*]*?)\b(fa_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", text):
        ret, name, params = " ".join(m.group(1).split()), m.group(2), " ".join(m.group(3).split())
        plist = [] if params in ("", "void") else [p.strip() for p in params.split(",")]
        decls[name] = (ret, plist)
    return decls


def _ctype(decl: str):
    """ctypes type of one C declaration (a parameter with its name, or a return type)."""
    d = decl.replace("const ", "").strip()
    if "*" in d:
        return ctypes.c_char_p if d.startswith("char") else ctypes.c_void_p
    base = d.split()[0]
    return {"int": ctypes.c_int, "float": ctypes.c_float, "size_t": ctypes.c_size_t,
            "unsigned": ctypes.c_uint}[base]


def test_every_declaration_matches_its_binding():
    decls = _declarations()
    assert set(decls) == set(_lib.SIGNATURES)
    for name, (ret, params) in decls.items():
        res, args = _lib.SIGNATURES[name]
        assert _ctype(ret) is res, (name, ret, res)
        assert len(args) == len(params), (name, len(args), len(params))
        for i, (p, a) in enumerate(zip(params, args)):
            assert _ctype(p) is a, (name, i, p, a)


def test_parser_sees_the_documented_calls():
    decls = _declarations()
    ret, params = decls["fa_fwd"]
    assert ret == "int" and len(params) == 13 and params[9].startswith("float")
    ret, params = decls["fa_bwd_workspace_size"]
    assert ret == "size_t" and len(params) == 4
    assert decls["fa_last_error"] == ("const char*", []) or decls["fa_last_error"][1] == []
