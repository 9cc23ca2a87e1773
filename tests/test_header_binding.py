"""The Python binding marshals exactly what include/lstm.h declares (CPU).

The ctypes binding is hand-written next to the C header; a parameter added,
dropped or reordered on one side only would pass pointers into the wrong
slots.  These checks parse the header and compare, for every exported call,
the parameter count and kind (pointer, size_t, int-like, 64-bit integer,
float), the field order and sizes of the two structs, and the constants.
"""
import ctypes
import os
import re

import pytest

from layer_lstm_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lstm.h")


def _header():
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    return re.sub(r"//[^\n]*", " ", text)


def _params(text, name):
    m = re.search(r"\b" + name + r"\s*\(([^;{]*?)\)\s*;", text)
    assert m, f"{name} not declared in include/lstm.h"
    body = " ".join(m.group(1).split())
    if body in ("", "void"):
        return []
    return [p.strip() for p in body.split(",")]


def _c_kind(param):
    if "*" in param or param.startswith("cudaStream_t"):
        return "ptr"
    t = param.rsplit(" ", 1)[0]
    if t == "size_t":
        return "size"
    if t in ("int", "lstm_status", "lstm_dtype"):
        return "int"
    if t in ("unsigned long long", "long long"):
        return "i64"
    if t == "float":
        return "float"
    raise AssertionError(f"unclassified parameter type: {param}")


def _ctypes_kind(t):
    if t in (ctypes.c_void_p, ctypes.c_char_p) or (isinstance(t, type) and issubclass(t, ctypes._Pointer)):
        return "ptr"
    if t is ctypes.c_size_t:
        return "size"
    if t is ctypes.c_int:
        return "int"
    if t in (ctypes.c_ulonglong, ctypes.c_longlong):
        return "i64"
    if t is ctypes.c_float:
        return "float"
    raise AssertionError(f"unclassified ctypes type: {t}")


@pytest.fixture(scope="module")
def lib():
    return binding.load()


@pytest.mark.parametrize("name", binding.EXPORTED)
def test_call_signatures_match_header(lib, name):
    params = _params(_header(), name)
    argtypes = getattr(lib, name).argtypes
    assert len(argtypes) == len(params), f"{name}: {len(argtypes)} ctypes args, header has {params}"
    for i, (p, t) in enumerate(zip(params, argtypes)):
        assert _c_kind(p) == _ctypes_kind(t), f"{name} arg {i} ({p}) bound as {t}"


def _struct_fields(text, name):
    m = re.search(r"typedef\s+struct\s*\{([^}]*)\}\s*" + name + r"\s*;", text)
    assert m, f"struct {name} not found"
    fields = []
    for decl in m.group(1).split(";"):
        decl = " ".join(decl.split())
        if decl:
            typ, field = decl.rsplit(" ", 1)
            fields.append((typ, field.lstrip("*"), "*" in decl))
    return fields


C_SIZES = {"int": 4, "lstm_dtype": 4, "float": 4, "double": 8, "long long": 8,
           "unsigned long long": 8}


@pytest.mark.parametrize("cname,pytype", [("lstm_desc", binding.lstm_desc),
                                          ("lstm_kernel_time", binding.lstm_kernel_time)])
def test_struct_layouts_match_header(cname, pytype):
    fields = _struct_fields(_header(), cname)
    assert [name for _, name, _ in fields] == [name for name, _ in pytype._fields_]
    for (typ, name, is_ptr), (pname, ptype) in zip(fields, pytype._fields_):
        size = ctypes.sizeof(ctypes.c_void_p) if is_ptr else C_SIZES[typ]
        assert ctypes.sizeof(ptype) == size, f"{cname}.{name}: {typ} vs {ptype}"


def test_constants_match_header():
    text = _header()
    consts = {k: int(v) for k, v in re.findall(r"\b(LSTM_[A-Z0-9_]+)\s*=\s*(\d+)", text)}
    for k, v in consts.items():
        assert getattr(binding, k) == v, k
    defines = dict(re.findall(r"#define\s+(LSTM_[A-Z0-9_]+)\s+(\d+)\s*$", text, flags=re.M))
    assert binding.LSTM_TRACE_MAX_STEPS == int(defines["LSTM_TRACE_MAX_STEPS"])
    assert binding.LSTM_TRACE_EVENTS == int(defines["LSTM_TRACE_EVENTS"])
    m = re.search(r"#define\s+LSTM_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", text)
    assert m and binding.LSTM_NOALLOC_SCRATCH_BYTES == int(m.group(1)) << int(m.group(2))
