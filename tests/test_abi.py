"""The C-ABI library: it loads, exports every entry point the public headers
declare, and its host-side argument checks work without a GPU."""
import ctypes
import os
import re

import pytest

import decode_megakernel_interpreter_b200 as mk

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in ("mk.h", "mk_host.h"):
        src = open(os.path.join(ROOT, "include", h)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"\b(mk_\w+)\s*\(", src))
    return sorted(names)


def test_every_declared_symbol_is_exported():
    lib = mk.load()
    names = declared_functions()
    assert {"mk_create", "mk_plan", "mk_decode_step", "mk_get_status", "mk_status_string",
            "mk_destroy"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    for code in range(-8, 1):
        assert mk.mk_status_string(code)
    assert mk.mk_status_string(-99) == "unknown status"
    assert "timed out" in mk.mk_status_string(mk.MK_ERR_TIMEOUT)


def test_null_arguments_rejected_without_gpu():
    lib = mk.load()
    h = ctypes.c_void_p()
    assert lib.mk_create(None, None, None, ctypes.byref(h)) == mk.MK_ERR_INVALID_ARG
    assert h.value is None
    assert lib.mk_plan(None, None) == mk.MK_ERR_INVALID_ARG
    assert lib.mk_decode_step(None, None, None, None, None, None) == mk.MK_ERR_INVALID_ARG
    assert lib.mk_get_status(None, None) == mk.MK_ERR_INVALID_ARG
    assert lib.mk_get_plan_info(None, None) == mk.MK_ERR_INVALID_ARG
    assert lib.mk_trace_read(None, None, 0) == mk.MK_ERR_INVALID_ARG
    lib.mk_destroy(None)


def test_unsupported_shape_rejected_before_any_device_call():
    import synth
    lib = mk.load()
    cfg = mk.make_config(synth.TINY, 1, 64)
    cfg.head_dim = 96
    w = mk.mk_weights()
    kv = mk.mk_kv_cache()
    h = ctypes.c_void_p()
    # null pointers are checked after the shape, so a bad shape wins
    assert lib.mk_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(kv), ctypes.byref(h)) == \
        mk.MK_ERR_UNSUPPORTED_SHAPE
    cfg = mk.make_config(synth.TINY, 1, 64)
    cfg.max_batch = 17
    assert lib.mk_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(kv), ctypes.byref(h)) == \
        mk.MK_ERR_UNSUPPORTED_SHAPE
    cfg = mk.make_config(synth.TINY, 1, 0)
    assert lib.mk_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(kv), ctypes.byref(h)) == \
        mk.MK_ERR_INVALID_ARG


def test_struct_layouts_match_headers():
    assert ctypes.sizeof(mk.mk_instr_desc) == 32
    assert ctypes.sizeof(mk.mk_config) == 56
    assert ctypes.sizeof(mk.mk_plan_opts) == 56


C_TYPES = {"int32_t": ctypes.c_int32, "int64_t": ctypes.c_int64, "uint32_t": ctypes.c_uint32,
           "uint16_t": ctypes.c_uint16, "uint8_t": ctypes.c_uint8, "float": ctypes.c_float,
           "double": ctypes.c_double}


def header_struct(name):
    """(field, C type) of `typedef struct { ... } name;` in the public headers
    (pointer fields typed "ptr")."""
    for h in ("mk.h", "mk_host.h"):
        src = open(os.path.join(ROOT, "include", h)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        m = re.search(r"typedef struct \{([^}]*)\}\s*" + name + r"\s*;", src)
        if m:
            out = []
            for decl in m.group(1).split(";"):
                decl = decl.strip()
                if not decl:
                    continue
                f = re.match(r"(?:const\s+)?(\w+)\s*(\*?)\s*(\w+(?:\s*,\s*\w+)*)$", decl)
                assert f, decl
                for fld in f.group(3).split(","):
                    out.append((fld.strip(), "ptr" if f.group(2) else f.group(1)))
            return out
    raise AssertionError(name)


@pytest.mark.parametrize("name", ["mk_config", "mk_plan_opts", "mk_plan_info", "mk_instr_desc", "mk_layer_weights",
                                  "mk_weights", "mk_kv_cache"])
def test_binding_structs_follow_the_headers(name):
    """Field names, order and types of the ctypes mirrors equal the C
    declarations (a field added on one side only fails here)."""
    want = header_struct(name)
    got = getattr(mk, name)._fields_
    assert [n for n, _ in got] == [n for n, _ in want]
    for (n, ct), (_, hc) in zip(got, want):
        if hc == "ptr":
            assert ct in (ctypes.c_void_p,) or issubclass(ct, ctypes._Pointer), n
        else:
            assert ct is C_TYPES[hc], (n, ct, hc)


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    """Without libmk.so there is no fallback: loading raises."""
    monkeypatch.setattr(mk, "_lib", None)
    with pytest.raises(ImportError):
        mk.load(str(tmp_path / "libmk.so"))


def test_product_code_never_imports_the_oracle():
    """The engine package and its sources name neither the oracle package nor
    its library (only tests, the smoke entry and the bench's CPU legs may)."""
    pkg = os.path.join(ROOT, "decode_megakernel_interpreter_b200")
    for dirpath, _, files in os.walk(pkg):
        if "_build" in dirpath:
            continue
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert not re.search(r"\bimport oracle\b|from oracle\b|liboracle|llama_oracle", src), f


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "mk.h"
#include "mk_host.h"

int main(void) {
  mk_handle *h = (mk_handle *)1;
  mk_config cfg;
  memset(&cfg, 0, sizeof cfg);
  if (mk_create(NULL, NULL, NULL, &h) != MK_ERR_INVALID_ARG || h != NULL) return 1;
  if (mk_plan(NULL, NULL) != MK_ERR_INVALID_ARG) return 2;
  if (mk_decode_step(NULL, NULL, NULL, NULL, NULL, NULL) != MK_ERR_INVALID_ARG) return 3;
  if (strcmp(mk_status_string(MK_OK), "ok") != 0) return 4;
  mk_destroy(NULL);
  printf("%zu %zu %zu\n", sizeof(mk_config), sizeof(mk_plan_opts), sizeof(mk_instr_desc));
  return 0;
}
"""


def test_headers_compile_as_c_and_link(tmp_path):
    """include/*.h are plain C: a C99 program includes them, links libmk.so
    and calls the argument checks (no GPU needed); struct sizes agree with
    the binding's."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    lib = mk.LIB_PATH
    src = tmp_path / "abi_check.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "abi_check"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                           "-o", str(exe), lib, "-Wl,-rpath," + os.path.dirname(lib)])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, (out.returncode, out.stderr)
    sizes = [int(x) for x in out.stdout.split()]
    assert sizes == [ctypes.sizeof(mk.mk_config), ctypes.sizeof(mk.mk_plan_opts), ctypes.sizeof(mk.mk_instr_desc)]
