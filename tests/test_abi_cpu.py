"""CPU-side checks of the C ABI: the library loads, exports every symbol
include/pkv.h declares, and rejects bad host arguments before touching the
GPU.  No compute call is made here."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"PKV_API\s+[\w\s\*]+?\b(\w+)\s*\(", src))
    return names


def test_header_declares_the_documented_calls():
    names = _declared()
    for n in ("pkv_pool_create", "pkv_append", "paged_attention_decode", "pkv_gather",
              "pkv_get_device_error", "pkv_decode_workspace_bytes"):
        assert n in names


def test_library_exports_every_declared_symbol():
    from paged_attention_decode_pkv_b200 import pkv
    lib = ctypes.CDLL(pkv.LIB_PATH)
    for n in _declared():
        assert hasattr(lib, n), n
    assert set(pkv.EXPORTS) >= _declared()


def test_status_strings():
    from paged_attention_decode_pkv_b200 import pkv
    assert pkv.status_string(0) == "ok"
    assert "outside the pool" in pkv.status_string(pkv.ERR_BAD_PAGE)
    assert pkv.status_string(12345) == "unknown status"
    assert "race" in pkv.status_string(pkv.ERR_APPEND_CONFLICT)


def test_binding_constants_match_the_header():
    """Every PKV_ERR_* code and PKV_LAUNCH_* flag of the header has the same
    value under the same name in the Python binding."""
    from paged_attention_decode_pkv_b200 import pkv
    src = open(os.path.join(ROOT, "include", "pkv.h")).read()
    errs = dict(re.findall(r"\bPKV_(ERR_\w+)\s*=\s*(-?\d+)", src))
    flags = dict(re.findall(r"#define\s+PKV_(LAUNCH_\w+)\s+(\(?[\d\s<]+\)?)", src))
    assert len(errs) >= 10 and len(flags) >= 5
    for name, value in list(errs.items()) + list(flags.items()):
        assert getattr(pkv, name) == eval(value), name


def test_pool_create_rejects_bad_shapes_and_null_out():
    from paged_attention_decode_pkv_b200 import pkv
    h = ctypes.c_void_p()
    assert pkv.lib.pkv_pool_create(16, 32, 8, 64, None, 0, ctypes.byref(h)) == pkv.ERR_UNSUPPORTED
    assert pkv.lib.pkv_pool_create(16, 16, 4, 64, None, 0, ctypes.byref(h)) == pkv.ERR_UNSUPPORTED
    assert pkv.lib.pkv_pool_create(16, 16, 8, 128, None, 0, ctypes.byref(h)) == pkv.ERR_UNSUPPORTED
    assert pkv.lib.pkv_pool_create(0, 16, 8, 64, None, 0, ctypes.byref(h)) == pkv.ERR_INVALID_ARG
    assert pkv.lib.pkv_pool_create(16, 16, 8, 64, None, 0, None) == pkv.ERR_INVALID_ARG
    # a pool whose TMA row coordinates would overflow int32
    assert pkv.lib.pkv_pool_create(1 << 23, 16, 8, 64, None, 0, ctypes.byref(h)) == \
        pkv.ERR_UNSUPPORTED


def test_calls_reject_null_pool():
    from paged_attention_decode_pkv_b200 import pkv
    P = ctypes.c_void_p(16)
    assert pkv.lib.pkv_append(None, P, P, P, P, 0, 1, 1, 1, None) == pkv.ERR_INVALID_ARG
    assert pkv.lib.paged_attention_decode(P, None, P, P, 0, 0.125, P, 1, 1, 1, P, 1 << 20,
                                          None) == pkv.ERR_INVALID_ARG
    assert pkv.lib.pkv_gather(None, P, P, 0, P, P, 1, 1, 1, 16, None) == pkv.ERR_INVALID_ARG
    n = ctypes.c_size_t()
    assert pkv.lib.pkv_decode_workspace_bytes(None, 4, ctypes.byref(n)) == pkv.ERR_INVALID_ARG
    assert pkv.lib.pkv_pool_destroy(None) == pkv.OK
    assert pkv.lib.pkv_pool_num_pages(None) == -1
    assert pkv.lib.pkv_fill(None, P, P, P, P, P, 16, 0, 1, 1, 1, None) == pkv.ERR_INVALID_ARG


def test_decode_params_struct_matches_the_header(tmp_path):
    # the binding's ctypes mirror of pkv_decode_params must have the C layout
    from paged_attention_decode_pkv_b200 import pkv
    import subprocess
    fields = [f[0] for f in pkv.DecodeParams._fields_]
    src = ["#include <stdio.h>", "#include <stddef.h>", '#include "pkv.h"', "int main(void) {",
           '  printf("%zu\\n", sizeof(pkv_decode_params));']
    src += ['  printf("%%zu\\n", offsetof(pkv_decode_params, %s));' % f for f in fields]
    src += ["  return 0;", "}"]
    (tmp_path / "layout.c").write_text("\n".join(src))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(tmp_path / "layout.c"),
                    "-o", str(exe)], check=True)
    got = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True,
                                          check=True).stdout.split()]
    assert got[0] == ctypes.sizeof(pkv.DecodeParams)
    assert got[1:] == [getattr(pkv.DecodeParams, f).offset for f in fields]
