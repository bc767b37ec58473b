"""include/csa2.h is a C header: a C11 program (tests/c_consumer.c) compiles
against it with -Wall -Wextra -Werror -pedantic, links libcsa2.so, and gets
the documented host-side statuses without a GPU (argument, shape and alignment
errors are returned before any CUDA call)."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "fp4_kv_cache_quantize_b200")

WANT = {
    "quantize_ch": 2, "quantize_null": 1, "quantize_empty": 0, "quantize_align": 3,
    "dequantize_null": 1, "index_full_kv": 1, "index_full_codes": 1, "reindex_kv": 1,
    "attn_kv": 1, "group_null": 1, "group_empty": 1, "group_ws_size": 0, "append_kv": 1,
    "cp_ws_bad": 0, "cp_rows_bad": 2, "cp_filter_unit": 1, "cp_partial_floats": 2 * 16 * 514,
}


@pytest.fixture(scope="module")
def consumer(tmp_path_factory):
    if not os.path.exists(os.path.join(LIBDIR, "libcsa2.so")):
        from fp4_kv_cache_quantize_b200 import build
        build.build()
    exe = str(tmp_path_factory.mktemp("c") / "c_consumer")
    subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
                           "-I" + os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "c_consumer.c"), "-L" + LIBDIR, "-lcsa2",
                           "-Wl,-rpath," + LIBDIR, "-o", exe])
    return exe


def test_c_program_sees_the_documented_statuses(consumer):
    out = subprocess.run([consumer], capture_output=True, text=True, timeout=120, check=True)
    got = {}
    for line in out.stdout.splitlines():
        k, v = line.split(" ", 1)
        got[k] = v
    for k, v in WANT.items():
        assert int(got[k]) == v, (k, got[k], v)
    assert got["status_string"] == "CSA2_ERR_TIMEOUT"
    assert got["constants"] == "512 16 8 64 8 128 512 2048 16"
