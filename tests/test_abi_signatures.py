"""The binding's ctypes signatures against the C declarations in include/*.h (host only):
every declared function has one argument type per parameter, a pointer where the header
has a pointer, and an integer or float of the header's width elsewhere. A mismatch would
pass garbage through the boundary without any error."""
import ctypes
import os
import re

import pytest

import nvfp4_kv_cache_kvq_b200 as kvq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", h) for h in ("kvq.h", "kvq_testing.h")]

# scalar C types -> (ctypes type, or "pointer")
SCALARS = {
    "int64_t": ctypes.c_int64, "int32_t": ctypes.c_int32, "uint64_t": ctypes.c_uint64,
    "uint32_t": ctypes.c_uint32, "float": ctypes.c_float, "kvq_scale_rule": ctypes.c_int32,
    "kvq_status": ctypes.c_int32, "int": ctypes.c_int,
}
POINTER_TYPEDEFS = {"kvq_stream_t"}


def _declarations():
    out = {}
    for path in HEADERS:
        src = open(path).read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        for m in re.finditer(r"\b(kvq_status|void|const\s+char\s*\*)\s+(kvq_\w+)\s*\(([^)]*)\)\s*;", src):
            params = [p.strip() for p in m.group(3).split(",")]
            if params == ["void"] or params == [""]:
                params = []
            out[m.group(2)] = (m.group(1), params)
    return out


def _kind(param: str):
    """'pointer', or the ctypes scalar type of one C parameter declaration."""
    decl = re.sub(r"\b\w+$", "", param).strip() if not param.endswith("*") else param
    if "*" in decl:
        return "pointer"
    base = decl.replace("const", "").strip()
    if base in POINTER_TYPEDEFS:
        return "pointer"
    return SCALARS[base]


def _is_pointer_ctype(t) -> bool:
    return t in (ctypes.c_void_p, ctypes.c_char_p) or (isinstance(t, type) and issubclass(t, ctypes._Pointer))


DECLS = _declarations()


def test_every_declaration_is_found():
    assert len(DECLS) >= 30
    for name in ("kvq_quantize", "kvq_append_batch", "kvq_attention", "kvq_device_status",
                 "kvq_quantize_launches", "kvq_testing_set_fused_wait"):
        assert name in DECLS


@pytest.mark.parametrize("name", sorted(DECLS))
def test_binding_signature_matches_header(name):
    lib = kvq.load()
    ret, params = DECLS[name]
    fn = getattr(lib, name)
    assert fn.argtypes is not None, f"{name}: no argtypes in the binding"
    assert len(fn.argtypes) == len(params), (name, len(fn.argtypes), params)
    for i, (t, p) in enumerate(zip(fn.argtypes, params)):
        kind = _kind(p)
        if kind == "pointer":
            assert _is_pointer_ctype(t), f"{name} arg {i} ({p}): header pointer, binding {t}"
        else:
            assert not _is_pointer_ctype(t) and ctypes.sizeof(t) == ctypes.sizeof(kind), (
                f"{name} arg {i} ({p}): header {kind.__name__}, binding {t}")
    if ret == "void":
        assert fn.restype is None
    elif "char" in ret:
        assert fn.restype is ctypes.c_char_p
    else:
        assert fn.restype in (ctypes.c_int, ctypes.c_int32)


def _structs():
    """typedef struct { fields } name; -> {name: [(field, 'pointer' or ctypes type)]}."""
    out = {}
    src = open(HEADERS[0]).read()
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    for m in re.finditer(r"typedef\s+struct\s*\{([^}]*)\}\s*(\w+)\s*;", src):
        fields = []
        for decl in m.group(1).split(";"):
            decl = decl.strip()
            if not decl:
                continue
            name = re.search(r"(\w+)$", decl).group(1)
            fields.append((name, _kind(decl)))
        out[m.group(2)] = fields
    return out


@pytest.mark.parametrize("c_name,py_struct", [("kvq_cache", "_Cache"), ("kvq_recent_cache", "_RecentCache")])
def test_binding_structs_match_header(c_name, py_struct):
    """Field order, kind and width of the cache views the binding passes by pointer."""
    want = _structs()[c_name]
    got = getattr(kvq, py_struct)._fields_
    assert [f for f, _ in got] == [f for f, _ in want]
    for (f, t), (_, k) in zip(got, want):
        if k == "pointer":
            assert _is_pointer_ctype(t), (c_name, f)
        else:
            assert not _is_pointer_ctype(t) and ctypes.sizeof(t) == ctypes.sizeof(k), (c_name, f)
