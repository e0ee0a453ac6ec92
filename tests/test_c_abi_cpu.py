"""The C ABI as a C program and the Python binding see it (no GPU needed).

- include/indexcache.h compiles as strict C99 and as C++17;
- a C program links against the library and makes calls that must return
  before any device access (tests/c_abi/abi_check.c);
- the binding's ctypes structures have the C layouts (sizes and offsets
  reported by the C compiler), and its argument/return types match every
  prototype of the header, so no argument is truncated or misplaced.
"""
import ctypes
import json
import os
import re
import shutil
import subprocess

import pytest

import cross_layer_top_full_b200 as ic
from cross_layer_top_full_b200 import build as icbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")
HEADER = os.path.join(INCLUDE, "indexcache.h")

pytestmark = pytest.mark.skipif(shutil.which("gcc") is None or shutil.which("g++") is None,
                                reason="needs gcc and g++")


@pytest.fixture(scope="module")
def libpath():
    if not os.path.exists(ic.library_path()):
        icbuild.build()
    return ic.library_path()


@pytest.fixture(scope="module")
def c_report(libpath, tmp_path_factory):
    out = tmp_path_factory.mktemp("c_abi")
    exe = str(out / "abi_check")
    libdir = os.path.dirname(libpath)
    subprocess.run(["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE,
                    os.path.join(ROOT, "tests", "c_abi", "abi_check.c"), "-L", libdir,
                    "-lindexcache", "-Wl,-rpath," + libdir, "-o", exe], check=True)
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stderr
    return json.loads(run.stdout)


@pytest.mark.parametrize("compiler,std", [("gcc", "-std=c99"), ("g++", "-std=c++17")])
def test_header_compiles_cleanly(tmp_path, compiler, std):
    src = tmp_path / ("h.c" if compiler == "gcc" else "h.cpp")
    src.write_text('#include "indexcache.h"\nint main(void) { return IC_OK; }\n')
    subprocess.run([compiler, std, "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE,
                    "-fsyntax-only", str(src)], check=True)


def test_c_client_calls_return_before_the_device(c_report):
    r = c_report
    assert r["version"] == ic.version()
    assert r["ok_string"] == "IC_OK"
    assert r["last_error_before"] == ""
    assert r["bad_pattern"] == -2 and r["short_pattern"] == -2   # IC_ERR_PATTERN
    assert r["bad_page_size"] == -1 and r["paged_no_ws"] == -4
    assert r["no_ws"] == -4          # IC_ERR_WORKSPACE: NULL workspace
    assert r["bad_k"] == -1          # IC_ERR_INVALID_ARG: k = 0
    assert r["workspace_size"] > 0
    assert r["launches"] == 0
    assert r["IC_STATUS_BYTES"] == ic.STATUS_BYTES


def _ctypes_layout(cls):
    return {name: getattr(cls, name).offset for name, _ in cls._fields_}


@pytest.mark.parametrize("cname,cls", [("ic_rows", ic.Rows), ("ic_stack_shape", ic.StackShape),
                                       ("ic_layer_io", ic.LayerIO),
                                       ("ic_paged_rows", ic.PagedRows)])
def test_binding_structs_have_the_c_layout(c_report, cname, cls):
    c = dict(c_report[cname])
    assert c.pop("size") == ctypes.sizeof(cls)
    assert c == _ctypes_layout(cls)


def test_enums_are_int_sized(c_report):
    # the binding passes ic_status / ic_dtype as c_int
    assert c_report["sizeof_enum"] == ctypes.sizeof(ctypes.c_int)


# ------------------------------------------------------------ prototypes vs binding
_SCALARS = {
    "int": ctypes.c_int, "ic_dtype": ctypes.c_int, "ic_status": ctypes.c_int,
    "int64_t": ctypes.c_int64, "size_t": ctypes.c_size_t, "float": ctypes.c_float,
    "uint64_t": ctypes.c_uint64, "ic_rows": ic.Rows,
}
_POINTEES = {"ic_stack_shape": ic.StackShape, "ic_layer_io": ic.LayerIO,
             "ic_paged_rows": ic.PagedRows, "int32_t": ctypes.c_int32}


def _prototypes():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = "\n".join(l for l in text.splitlines() if not l.lstrip().startswith("#"))
    protos = {}
    for m in re.finditer(r"([A-Za-z_][\w\s\*]*?)\b(ic_[a-z0-9_]+)\s*\(([^()]*)\)\s*;", text):
        ret, name, params = m.group(1), m.group(2), m.group(3).strip()
        args = []
        if params != "void":
            for p in params.split(","):
                p = re.sub(r"\b[A-Za-z_]\w*\s*$", "", p.strip())  # drop the parameter name
                args.append(" ".join(p.replace("*", " * ").split()))
        protos[name] = (" ".join(ret.replace("*", " * ").split()), args)
    return protos


def _compatible(ctype_text, ct):
    words = ctype_text.replace("const", " ").split()
    if "*" in words:
        base = [w for w in words if w != "*"][0]
        depth = words.count("*")
        if base == "char" and depth == 1:
            return ct is ctypes.c_char_p
        if depth == 1 and base in _POINTEES:
            return ct is ctypes.c_void_p or ct is ctypes.POINTER(_POINTEES[base])
        return ct is ctypes.c_void_p or (depth == 2 and ct is ctypes.POINTER(ctypes.c_void_p))
    (base,) = words
    return ct is _SCALARS[base]


def test_binding_signatures_match_the_header(libpath):
    ic.lib()
    sig = ic._SIG
    protos = _prototypes()
    assert len(protos) >= 15
    assert set(protos) == set(sig), set(protos) ^ set(sig)
    for name, (ret, args) in protos.items():
        res, argtypes = sig[name]
        assert _compatible(ret, res), (name, ret, res)
        assert len(args) == len(argtypes), (name, args, argtypes)
        for i, (a, t) in enumerate(zip(args, argtypes)):
            assert _compatible(a, t), (name, i, a, t)
