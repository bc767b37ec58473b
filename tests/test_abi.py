"""The C ABI library: it loads without a GPU and exports every entry point
that include/csa2.h declares; host-only entry points behave on the CPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa2.h")
LIB = os.path.join(ROOT, "fp4_kv_cache_quantize_b200", "libcsa2.so")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w\s\*]*?\b(csa2_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        from fp4_kv_cache_quantize_b200 import build
        build.build()
    return ctypes.CDLL(LIB)


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("csa2_quantize_fp4", "csa2_dequantize_fp4", "csa2_index_full",
                 "csa2_index_reindex", "csa2_sparse_attn_decode", "csa2_layer_group",
                 "csa2_status_string", "csa2_last_error", "csa2_sync_status"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings_and_host_side_errors(lib):
    lib.csa2_status_string.restype = ctypes.c_char_p
    lib.csa2_last_error.restype = ctypes.c_char_p
    assert lib.csa2_status_string(0) == b"CSA2_OK"
    assert lib.csa2_status_string(6) == b"CSA2_ERR_TIMEOUT"
    # shape errors are caught on the host before any CUDA call
    lib.csa2_quantize_fp4.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    assert lib.csa2_quantize_fp4(None, 4, 24, None, None, None) == 2
    assert b"multiple of 16" in lib.csa2_last_error()
    assert lib.csa2_quantize_fp4(None, 0, 512, None, None, None) == 0     # nothing to do
    assert lib.csa2_quantize_fp4(None, 4, 512, None, None, None) == 1     # NULL input
    assert lib.csa2_quantize_fp4(ctypes.c_void_p(16 * 3 + 8), 4, 512, ctypes.c_void_p(64),
                                 ctypes.c_void_p(64), None) == 3          # misaligned


def test_group_host_validation(lib):
    from fp4_kv_cache_quantize_b200 import csa2
    lib2 = csa2._lib
    desc = csa2.GroupDesc()
    desc.n_layers = 1
    assert lib2.csa2_layer_group(ctypes.byref(desc), None, 0, None) != 0
    assert lib2.csa2_group_workspace_size(ctypes.byref(desc)) == 0
