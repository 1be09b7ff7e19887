"""The ctypes binding declares every C-ABI entry point with the parameter
list the header gives it: the same number of parameters, pointers where the
header has pointers, size_t and int where it has those."""
import ctypes
import os
import re

import pytest

import mamba_ssd_sequence_b200 as ssd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declarations():
    text = open(os.path.join(ROOT, "include", "ssd.h")).read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    decls = {}
    for m in re.finditer(r"([A-Za-z_][\w \*]*?)\b(ssd_\w+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S):
        params = [p.strip() for p in m.group(3).split(",") if p.strip() and p.strip() != "void"]
        decls[m.group(2)] = params
    return decls


def _kind_of_param(p):
    if "*" in p:
        return "ptr"
    if "size_t" in p:
        return "size"
    if "long long" in p:
        return "int64"
    return "int"


def _kind_of_argtype(t):
    if t is ctypes.c_void_p or (isinstance(t, type) and issubclass(t, ctypes._Pointer)):
        return "ptr"
    if t is ctypes.c_size_t:
        return "size"
    if t is ctypes.c_int:
        return "int"
    if t is ctypes.c_longlong:
        return "int64"
    return repr(t)


def test_binding_argtypes_match_header():
    try:
        lib = ssd.load_library()
    except (OSError, RuntimeError) as e:  # the library is built by build(); a CPU-only box may lack CUDA
        pytest.skip(f"library not loadable here: {e}")
    decls = _declarations()
    assert len(decls) >= 14, sorted(decls)
    checked = 0
    for name, params in decls.items():
        fn = getattr(lib, name)
        if fn.argtypes is None:
            continue
        assert len(fn.argtypes) == len(params), name
        assert [_kind_of_argtype(t) for t in fn.argtypes] == [_kind_of_param(p) for p in params], name
        checked += 1
    assert checked >= 12
