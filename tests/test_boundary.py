"""The product's boundaries, checked statically on the CPU:
  * the Python binding binds every entry point that include/csa2.h declares,
    under the same name, and exposes a wrapper of that name;
  * the shape constants of the binding are the header's;
  * nothing in the package (Python or CUDA) imports, links or names the
    oracle's code, and the oracle imports or includes nothing of the package."""
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "fp4_kv_cache_quantize_b200")
HEADER = os.path.join(ROOT, "include", "csa2.h")


def _header():
    return re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)


def test_binding_covers_every_declared_entry_point():
    names = set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(csa2_\w+)\s*\(", _header(), flags=re.M))
    src = open(os.path.join(PKG, "csa2.py")).read()
    bound = set(re.findall(r'_sig\("(csa2_\w+)"', src))
    wrappers = set(re.findall(r"^def (csa2_\w+)\(", src, flags=re.M))
    assert names - bound == set(), sorted(names - bound)
    # every entry point but the string helpers and the trace hook has a wrapper
    helpers = {"csa2_status_string", "csa2_last_error"}
    assert names - wrappers - helpers == set(), sorted(names - wrappers - helpers)


def test_binding_constants_are_the_headers():
    from fp4_kv_cache_quantize_b200 import csa2
    enum = dict((k, v) for k, v in re.findall(r"\b(CSA2_[A-Z_]+)\s*=\s*([^,/\n]+)", _header()))
    val = lambda s: eval(s.strip(), {})  # noqa: E731  (integer literals and shifts)
    assert val(enum["CSA2_D"]) == csa2.D and val(enum["CSA2_H"]) == csa2.H
    assert val(enum["CSA2_HI"]) == csa2.HI and val(enum["CSA2_DI"]) == csa2.DI
    assert val(enum["CSA2_BLK"]) == csa2.BLK and val(enum["CSA2_W"]) == csa2.W
    assert val(enum["CSA2_MAX_TOPK"]) == csa2.MAX_TOPK
    assert val(enum["CSA2_MAX_POOL"]) == csa2.MAX_POOL
    assert val(enum["CSA2_MAX_ROWS"]) == csa2.MAX_ROWS
    assert (csa2.FULL, csa2.REINDEX, csa2.REUSE) == (0, 1, 2)
    status = dict(re.findall(r"\b(CSA2_(?:OK|ERR_[A-Z_]+))\s*=\s*(\d+)", _header()))
    assert {int(v): k for k, v in status.items()} == csa2.STATUS


def test_product_and_oracle_share_nothing():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if not f.endswith((".py", ".cu", ".cuh", ".h")):
                continue
            text = open(os.path.join(dirpath, f)).read()
            assert not re.search(r"^\s*(import oracle|from oracle)", text, flags=re.M), f
            assert "csa2_oracle" not in text and "csa2o_" not in text, f
    odir = os.path.join(ROOT, "oracle")
    for f in os.listdir(odir):
        if f.endswith((".c", ".h", ".py")):
            text = open(os.path.join(odir, f)).read()
            assert not re.search(r"^\s*(import|from)\s+fp4_kv_cache_quantize_b200", text,
                                 flags=re.M), f
            assert not re.search(r'#include\s*["<][^">]*(csrc|csa2\.h|kernels\.h)', text), f
