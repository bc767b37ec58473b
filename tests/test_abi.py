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


def test_cp_host_validation(lib):
    """Shard and argument checks of the context-parallel entry points run on
    the host, before any CUDA call."""
    from fp4_kv_cache_quantize_b200 import csa2
    lib2 = csa2._lib
    bad = [csa2.CpShard(0, 2, 100), csa2.CpShard(2, 2, 128), csa2.CpShard(-1, 2, 128),
           csa2.CpShard(0, 17, 128), csa2.CpShard(0, 2, 1 << 20), csa2.CpShard(0, 0, 128)]
    for sh in bad:
        assert csa2.csa2_cp_workspace_size(sh, 1, 1, 512) == 0
        assert lib2.csa2_cp_local_rows(ctypes.byref(sh), None, 1, None, None, 0, None) != 0
    assert lib2.csa2_cp_local_rows(None, None, 1, None, None, 0, None) == 1
    assert csa2.csa2_cp_partial_floats(2, 20) == 20 * 2 * 16 * 514
    assert csa2.csa2_cp_partial_floats(0, 20) == 0
    sh = csa2.CpShard(0, 2, 128)
    p = ctypes.c_void_p(256)
    f = lib2.csa2_cp_filter
    # unit other than 1 or 8
    assert f(ctypes.byref(sh), 3, p, p, 1, 1, p, p, 1, None, None, p, 256, None) == 1
    # copy without copy_count
    assert f(ctypes.byref(sh), 1, p, p, 1, 1, p, p, 1, p, None, p, 256, None) == 1
    # stride beyond the pool bound
    assert f(ctypes.byref(sh), 1, p, p, 4096, 1, p, p, 1, None, None, p, 256, None) == 2
    # misaligned count array
    assert f(ctypes.byref(sh), 1, p, ctypes.c_void_p(258), 1, 1, p, p, 1, None, None, p, 256,
             None) == 3
    m = lib2.csa2_cp_select_merge
    assert m(ctypes.byref(sh), p, 1, 1, 1, 512, p, p, p, 256, None) == 1   # job >= n_jobs
    assert m(ctypes.byref(sh), ctypes.c_void_p(260), 1, 0, 1, 512, p, p, p, 256, None) == 3
    assert m(ctypes.byref(sh), p, 1, 0, 1, 513, p, p, p, 256, None) == 2   # top_k > 512


def test_cp_batched_host_validation(lib):
    """The batched context-parallel calls check their job and layer tables on
    the host, before any CUDA call."""
    from fp4_kv_cache_quantize_b200 import csa2
    lib2 = csa2._lib
    sh = csa2.CpShard(0, 2, 128)
    p = ctypes.c_void_p(256)
    i32 = lambda *v: (ctypes.c_int32 * len(v))(*v)  # noqa: E731
    fl = lib2.csa2_cp_filter_layers
    assert fl(ctypes.byref(sh), 0, i32(0), p, p, 512, 1, p, p, p, 256, None) == 2   # no layers
    assert fl(ctypes.byref(sh), 33, i32(*range(33)), p, p, 512, 1, p, p, p, 256, None) == 2
    assert fl(ctypes.byref(sh), 2, None, p, p, 512, 1, p, p, p, 256, None) == 1     # no table
    # a layer reading a later layer, and one reading a layer that reads another
    assert fl(ctypes.byref(sh), 3, i32(0, 2, 2), p, p, 512, 1, p, p, p, 256, None) == 1
    assert fl(ctypes.byref(sh), 3, i32(0, 0, 1), p, p, 512, 1, p, p, p, 256, None) == 1
    assert fl(ctypes.byref(sh), 2, i32(0, 0), p, p, 4096, 1, p, p, p, 256, None) == 2  # stride
    mj = lib2.csa2_cp_select_merge_jobs
    assert mj(ctypes.byref(sh), p, 0, i32(0), 4, 1, 512, p, p, p, 256, None) == 2    # no jobs
    assert mj(ctypes.byref(sh), p, 9, i32(*range(9)), 9, 1, 512, p, p, p, 256, None) == 2
    assert mj(ctypes.byref(sh), p, 2, i32(0, 4), 4, 1, 512, p, p, p, 256, None) == 1  # layer 4
    assert mj(ctypes.byref(sh), p, 1, None, 4, 1, 512, p, p, p, 256, None) == 1
    assert mj(ctypes.byref(sh), p, 1, i32(0), 4, 1, 513, p, p, p, 256, None) == 2    # top_k
    lj = lib2.csa2_cp_select_local_jobs
    assert lj(ctypes.byref(sh), None, 1, i32(0), 4, p, p, p, p, 512, 512, p, p, 256, None) == 1
    kv = csa2.KVView()
    assert lj(ctypes.byref(sh), ctypes.byref(kv), 9, i32(*range(9)), 9, p, p, p, p, 512, 512, p,
              p, 256, None) == 2
    assert lj(ctypes.byref(sh), ctypes.byref(kv), 1, i32(5), 4, p, p, p, p, 512, 512, p, p,
              256, None) == 1



def test_noalloc_checks_arguments_before_its_scratch_size():
    """csa2_index_full_noalloc validates the view and sizes like
    csa2_index_full, so a bad shape reports CSA2_ERR_SHAPE rather than a
    scratch-size error, and nothing is enqueued (no GPU here)."""
    from fp4_kv_cache_quantize_b200 import csa2
    lib2 = csa2._lib
    p = ctypes.c_void_p(256)
    kv = csa2.KVView()
    kv.codes = kv.scales = kv.idx_k = kv.n_rows = p
    kv.batch, kv.max_rows, kv.seq_stride, kv.pool_rows = -3, 1024, 1024, 1024
    f = lib2.csa2_index_full_noalloc
    args = (p, p, 512, 2048, p, p, p, p, None)
    assert f(ctypes.byref(kv), *args) == 2          # negative batch: a shape error
    kv.batch, kv.max_rows = 1, -5
    assert f(ctypes.byref(kv), *args) == 2          # negative max_rows: a shape error
    kv.max_rows = 1024
    assert f(ctypes.byref(kv), p, p, 0, 2048, p, p, p, p, None) == 2     # top_k = 0
    assert f(ctypes.byref(kv), p, None, 512, 2048, p, p, p, p, None) == 1  # NULL weights
    kv.batch, kv.max_rows, kv.seq_stride, kv.pool_rows = 8, 1 << 20, 1 << 20, 8 << 20
    assert f(ctypes.byref(kv), *args) == 4          # 8 x 1M positions: beyond the scratch
