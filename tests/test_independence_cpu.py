"""The oracle and the CUDA path share no code: the product package never imports
or loads oracle/, the oracle never imports the product package or includes a
header of the CUDA side, and the oracle's ctypes declarations match its C
prototypes (a mismatch would corrupt every comparison silently)."""
import ast
import ctypes
import os
import re

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "causal_flash_attention_attn_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _files(top, exts):
    for d, _, names in os.walk(top):
        for n in names:
            if n.endswith(exts):
                yield os.path.join(d, n)


def _imports(path):
    tree = ast.parse(open(path).read())
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            yield from (a.name for a in node.names)
        elif isinstance(node, ast.ImportFrom):
            yield node.module or ""


def test_product_never_imports_or_loads_the_oracle():
    for path in _files(PKG, (".py",)):
        mods = list(_imports(path))
        assert not any(m == "oracle" or m.startswith("oracle.") for m in mods), (path, mods)
        text = open(path).read()
        assert "attn_ref" not in text and "liboracle" not in text, path
    for path in _files(PKG, (".cu", ".cuh", ".h")):
        assert "oracle" not in re.sub(r"//.*|/\*.*?\*/", "", open(path).read(), flags=re.S), path


def test_oracle_never_imports_the_product_or_includes_its_headers():
    for path in _files(ORACLE, (".py",)):
        mods = list(_imports(path))
        assert not any(m.startswith("causal_flash_attention_attn_b200") for m in mods), (path, mods)
    for path in _files(ORACLE, (".c", ".h")):
        incs = re.findall(r'#include\s*[<"]([^>"]+)[>"]', open(path).read())
        assert all(i in ("math.h", "stdint.h", "stdlib.h", "string.h", "omp.h") for i in incs), (path, incs)


def _c_kind(decl):
    decl = " ".join(decl.replace("const ", "").split())
    if "*" in decl:
        return "ptr"
    return {"int": "int", "long": "long", "double": "double", "void": "void"}[decl.split()[0]]


def _ct_kind(t):
    if t is None:
        return "void"
    if t in (ctypes.c_int,):
        return "int"
    if t in (ctypes.c_long,):
        return "long"
    if t in (ctypes.c_double,):
        return "double"
    if isinstance(t, type) and issubclass(t, ctypes._Pointer) or t in (ctypes.c_void_p, ctypes.c_char_p):
        return "ptr"
    raise AssertionError(t)


def test_oracle_ctypes_declarations_match_the_c_prototypes():
    src = re.sub(r"/\*.*?\*/|//[^\n]*", " ", open(os.path.join(ORACLE, "attn_ref.c")).read(), flags=re.S)
    protos = {}
    for ret, name, params in re.findall(r"^(void|int|double|long)\s+(oracle_\w+)\s*\(([^)]*)\)\s*\{", src, flags=re.M):
        plist = [p.strip() for p in " ".join(params.split()).split(",")] if params.strip() not in ("", "void") else []
        protos[name] = (ret, [_c_kind(re.sub(r"\b\w+$", "", p).strip() or p) for p in plist])
    lib = oracle._load()
    checked = 0
    for name, (ret, kinds) in protos.items():
        fn = getattr(lib, name)
        if fn.argtypes is None:
            continue  # not called from Python
        assert [_ct_kind(t) for t in fn.argtypes] == kinds, name
        if ret == "int":
            assert fn.restype is ctypes.c_int, name   # void returns are never read
        checked += 1
    assert checked >= 8, protos.keys()
