import ctypes
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built libcsa2.so")
    config.addinivalue_line("markers", "slow: full-size workloads")


@pytest.fixture(scope="session")
def fmt_ref(tmp_path_factory):
    """ctypes handle on tests/fmt_ref.cpp (CUDA host conversion routines)."""
    out = tmp_path_factory.mktemp("fmtref") / "libfmtref.so"
    src = os.path.join(ROOT, "tests", "fmt_ref.cpp")
    inc = os.environ.get("CUDA_HOME", "/usr/local/cuda") + "/include"
    subprocess.check_call(["g++", "-O1", "-std=c++17", "-fPIC", "-shared", "-I" + inc,
                           "-o", str(out), src])
    lib = ctypes.CDLL(str(out))
    lib.ref_e4m3_satfinite.restype = ctypes.c_ubyte
    lib.ref_e4m3_satfinite.argtypes = [ctypes.c_float]
    lib.ref_e2m1_rn.restype = ctypes.c_ubyte
    lib.ref_e2m1_rn.argtypes = [ctypes.c_float]
    lib.ref_e2m1_value.restype = ctypes.c_float
    lib.ref_e2m1_value.argtypes = [ctypes.c_ubyte]
    lib.ref_e4m3_value.restype = ctypes.c_float
    lib.ref_e4m3_value.argtypes = [ctypes.c_ubyte]
    return lib


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle
