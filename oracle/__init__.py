"""CPU oracle for the CSA2 decode step over an FP4 global KV cache.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(``libcsa2.so`` and ``fp4_kv_cache_quantize_b200``) never imports it and shares
no code, header or table with it.

The arithmetic lives in ``csa2_oracle.c`` (plain single-threaded C, fp64 on
exactly decoded values, selections by full sort); this module only builds it
with gcc and marshals numpy arrays through ctypes.  Parity status of each
function, and the passages it follows, are in the C header.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csa2_oracle.c")
LIB = os.path.join(HERE, "libcsa2_oracle.so")

FULL, REINDEX, REUSE = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < max(
        os.path.getmtime(SRC), os.path.getmtime(os.path.join(HERE, "csa2_oracle.h"))
    ):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
             "-fno-fast-math", "-o", tmp, SRC, "-lm"]
        )
        os.replace(tmp, LIB)
    return LIB


class _KV(C.Structure):
    _fields_ = [("codes", C.c_void_p), ("scales", C.c_void_p), ("idxk", C.c_void_p),
                ("page_table", C.c_void_p), ("page_rows", C.c_int32),
                ("max_pages", C.c_int32), ("seq_stride", C.c_int64),
                ("pool_rows", C.c_int64)]


class _Dims(C.Structure):
    _fields_ = [("d", C.c_int32), ("h", C.c_int32), ("hi", C.c_int32),
                ("di", C.c_int32), ("blk", C.c_int32), ("w", C.c_int32)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        L = _lib
        L.csa2o_bf16_value.restype = C.c_double
        L.csa2o_bf16_value.argtypes = [C.c_uint16]
        L.csa2o_bf16_round.restype = C.c_uint16
        L.csa2o_bf16_round.argtypes = [C.c_double]
        L.csa2o_e2m1_value.restype = C.c_double
        L.csa2o_e2m1_value.argtypes = [C.c_uint8]
        L.csa2o_e4m3_value.restype = C.c_double
        L.csa2o_e4m3_value.argtypes = [C.c_uint8]
        L.csa2o_e2m1_encode.restype = C.c_uint8
        L.csa2o_e2m1_encode.argtypes = [C.c_float]
        L.csa2o_e4m3_encode.restype = C.c_uint8
        L.csa2o_e4m3_encode.argtypes = [C.c_float]
        L.csa2o_quantize_fp4.argtypes = [C.c_void_p, C.c_int64, C.c_int32, C.c_void_p, C.c_void_p]
        L.csa2o_dequantize_fp4.argtypes = [C.c_void_p, C.c_void_p, C.c_int64, C.c_int32, C.c_void_p]
        L.csa2o_row_of.restype = C.c_int64
        L.csa2o_row_of.argtypes = [C.POINTER(_KV), C.c_int32, C.c_int64]
        L.csa2o_scores.argtypes = [C.POINTER(_KV), C.POINTER(_Dims), C.c_int32, C.c_int64,
                                   C.c_void_p, C.c_void_p, C.c_void_p]
        L.csa2o_block_max.argtypes = [C.c_void_p, C.c_int64, C.c_int32, C.c_void_p]
        L.csa2o_select_topk.restype = C.c_int64
        L.csa2o_select_topk.argtypes = [C.c_void_p, C.c_void_p, C.c_int64, C.c_int64, C.c_void_p]
        L.csa2o_pool.restype = C.c_int64
        L.csa2o_pool.argtypes = [C.c_void_p, C.c_int64, C.c_int32, C.c_void_p]
        L.csa2o_attention.argtypes = [C.POINTER(_KV), C.POINTER(_Dims), C.c_int32, C.c_void_p,
                                      C.c_void_p, C.c_int32, C.c_void_p, C.c_int32,
                                      C.c_double, C.c_void_p]
        L.csa2o_layer_group.argtypes = [C.POINTER(_KV), C.POINTER(_Dims), C.c_int32, C.c_void_p,
                                        C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p,
                                        C.c_void_p, C.c_void_p, C.c_void_p, C.c_int32,
                                        C.c_int32, C.c_double, C.c_void_p, C.c_void_p,
                                        C.c_void_p, C.c_void_p, C.c_void_p]
        L.csa2o_layer_group_multi.argtypes = [C.POINTER(_KV), C.POINTER(_Dims), C.c_int32,
                                              C.c_int32, C.c_void_p, C.c_int32, C.c_void_p,
                                              C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                              C.c_void_p, C.c_int32, C.c_int32, C.c_double,
                                              C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                              C.c_void_p]
        L.csa2o_project_idxk.argtypes = [C.c_void_p, C.c_void_p, C.c_int32, C.c_int32,
                                         C.c_void_p]
        L.csa2o_cache_append.argtypes = [C.POINTER(_KV), C.POINTER(_Dims), C.c_int32,
                                         C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                         C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p,
                                         C.c_void_p, C.c_void_p, C.c_void_p]
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ------------------------------------------------------------------ formats
def bf16_value(bits: int) -> float:
    return lib().csa2o_bf16_value(int(bits))


def bf16_round(v: float) -> int:
    return lib().csa2o_bf16_round(float(v))


def bf16_round_array(v: np.ndarray) -> np.ndarray:
    f = lib().csa2o_bf16_round
    flat = np.asarray(v, dtype=np.float64).ravel()
    return np.array([f(float(x)) for x in flat], dtype=np.uint16).reshape(np.shape(v))


def e2m1_value(code: int) -> float:
    return lib().csa2o_e2m1_value(int(code))


def e4m3_value(bits: int) -> float:
    return lib().csa2o_e4m3_value(int(bits))


def e2m1_encode(q: float) -> int:
    return lib().csa2o_e2m1_encode(float(q))


def e4m3_encode(t: float) -> int:
    return lib().csa2o_e4m3_encode(float(t))


# ---------------------------------------------------------------- A1 / A2
def quantize_fp4(x_bf16: np.ndarray):
    """bf16 bits [rows, ch] -> (codes u8 [rows, ch/2], scales u8 [rows, ch/16])."""
    x = _c(x_bf16, np.uint16)
    rows, ch = x.shape
    codes = np.zeros((rows, ch // 2), np.uint8)
    scales = np.zeros((rows, ch // 16), np.uint8)
    rc = lib().csa2o_quantize_fp4(_p(x), rows, ch, _p(codes), _p(scales))
    if rc:
        raise ValueError("oracle quantize: bad arguments")
    return codes, scales


def dequantize_fp4(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    rows, half = codes.shape
    y = np.zeros((rows, half * 2), np.float64)
    rc = lib().csa2o_dequantize_fp4(_p(codes), _p(scales), rows, half * 2, _p(y))
    if rc:
        raise ValueError("oracle dequantize: bad arguments")
    return y


# -------------------------------------------------------------- KV views
class KV:
    """Row pools of the main KV (codes, scales), indexer K and the row map."""

    def __init__(self, codes, scales, idxk, *, seq_stride=0, page_table=None,
                 page_rows=64):
        self.codes = _c(codes, np.uint8)
        self.scales = _c(scales, np.uint8)
        self.idxk = _c(idxk, np.uint16)
        self.page_table = None if page_table is None else _c(page_table, np.int32)
        self.s = _KV(_p(self.codes), _p(self.scales), _p(self.idxk),
                     _p(self.page_table), page_rows,
                     0 if page_table is None else self.page_table.shape[1],
                     seq_stride, self.codes.shape[0])

    def row_of(self, b: int, p: int) -> int:
        return lib().csa2o_row_of(C.byref(self.s), b, p)


def dims(d=512, h=16, hi=8, di=64, blk=8, w=128):
    return _Dims(d, h, hi, di, blk, w)


def scores(kv: KV, dm, b: int, C_: int, q_idx, w) -> np.ndarray:
    q_idx = _c(q_idx, np.uint16)
    w = _c(w, np.float32)
    s = np.zeros(max(C_, 1), np.float64)
    rc = lib().csa2o_scores(C.byref(kv.s), C.byref(dm), b, C_, _p(q_idx), _p(w), _p(s))
    if rc:
        raise ValueError("oracle scores: row outside the pool")
    return s[:C_]


def block_max(s: np.ndarray, blk: int) -> np.ndarray:
    s = _c(s, np.float64)
    n = (len(s) + blk - 1) // blk
    bm = np.zeros(max(n, 1), np.float64)
    lib().csa2o_block_max(_p(s), len(s), blk, _p(bm))
    return bm[:n]


def select_topk(v: np.ndarray, k: int, ids: np.ndarray | None = None) -> np.ndarray:
    v = _c(v, np.float64)
    ids_c = None if ids is None else _c(ids, np.int64)
    out = np.zeros(max(min(k, len(v)), 1), np.int32)
    m = lib().csa2o_select_topk(_p(v), _p(ids_c), len(v), k, _p(out))
    return out[:m]


def pool(bm: np.ndarray, pool_blocks: int) -> np.ndarray:
    bm = _c(bm, np.float64)
    out = np.zeros(max(min(pool_blocks, len(bm)), 1), np.int32)
    m = lib().csa2o_pool(_p(bm), len(bm), pool_blocks, _p(out))
    return out[:m]


def attention(kv: KV, dm, b: int, q, idx, swa, swa_len: int, sm_scale: float):
    q = _c(q, np.uint16)
    idx = _c(idx, np.int32)
    swa = _c(swa, np.uint8)
    out = np.zeros((dm.h, dm.d), np.float64)
    rc = lib().csa2o_attention(C.byref(kv.s), C.byref(dm), b, _p(q), _p(idx), len(idx),
                               _p(swa), swa_len, sm_scale, _p(out))
    if rc:
        raise ValueError("oracle attention: row outside the pool")
    return out


def layer_group(kv: KV, dm, n_rows, modes, q_idx, w, q, swa, swa_len, *, top_k=512,
                pool_blocks=2048, sm_scale=None):
    """Run a CSA2 layer group; returns dict(idx, idx_count, pool, pool_count, out)."""
    n_rows = _c(n_rows, np.int64)
    modes = _c(modes, np.int32)
    q_idx = _c(q_idx, np.uint16)
    w = _c(w, np.float32)
    q = _c(q, np.uint16)
    swa = _c(swa, np.uint8)
    swa_len = _c(swa_len, np.int32)
    B, L = len(n_rows), len(modes)
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(dm.d)
    idx = np.full((L, B, top_k), -1, np.int32)
    idx_count = np.zeros((L, B), np.int32)
    pb = max(pool_blocks, 1)
    pool_ = np.full((B, pb), -1, np.int32)
    pool_count = np.zeros(B, np.int32)
    out = np.zeros((L, B, dm.h, dm.d), np.float64)
    rc = lib().csa2o_layer_group(C.byref(kv.s), C.byref(dm), B, _p(n_rows), L, _p(modes),
                                 _p(q_idx), _p(w), _p(q), _p(swa), _p(swa_len), top_k,
                                 pool_blocks, sm_scale, _p(idx), _p(idx_count), _p(pool_),
                                 _p(pool_count), _p(out))
    if rc:
        raise ValueError("oracle layer group: bad arguments or row outside the pool")
    return dict(idx=idx, idx_count=idx_count, pool=pool_[:, :pool_blocks],
                pool_count=pool_count, out=out)


# ---------------------------------------------------- cache append (next row)
def project_idxk(x_bf16: np.ndarray, w_idx: np.ndarray) -> np.ndarray:
    """bf16 indexer-K row of one bf16 main-KV entry (fp64 sum, bf16 RNE)."""
    x = _c(x_bf16, np.uint16)
    w = _c(w_idx, np.uint16)
    d, di = w.shape
    out = np.zeros(di, np.uint16)
    if lib().csa2o_project_idxk(_p(x), _p(w), d, di, _p(out)):
        raise ValueError("oracle project_idxk: bad arguments")
    return out


def cache_append(kv: KV, dm, n_rows: np.ndarray, x: np.ndarray, w_idx: np.ndarray,
                 x_swa: np.ndarray | None = None, swa: np.ndarray | None = None,
                 swa_pos: np.ndarray | None = None, swa_len: np.ndarray | None = None) -> int:
    """Append one step's entries in place: kv.codes/scales/idxk rows, n_rows
    (int64), and the window rings swa[L][B][w][d] with swa_pos (int64) and
    swa_len (int32).  Returns the oracle's return code (1 when a sequence's
    row is not mapped; that sequence is skipped)."""
    B = len(n_rows)
    for a, dt in ((n_rows, np.int64), (x, np.uint16), (w_idx, np.uint16)):
        if a.dtype != dt or not a.flags.c_contiguous:
            raise TypeError("cache_append: arrays must be C-contiguous of the documented dtype")
    L = 0 if x_swa is None else x_swa.shape[0]
    if L:
        for a, dt in ((x_swa, np.uint16), (swa, np.uint8), (swa_pos, np.int64),
                      (swa_len, np.int32)):
            if a.dtype != dt or not a.flags.c_contiguous:
                raise TypeError("cache_append: arrays must be C-contiguous of the documented dtype")
    return lib().csa2o_cache_append(C.byref(kv.s), C.byref(dm), B, _p(kv.codes), _p(kv.scales),
                                    _p(kv.idxk), _p(n_rows), _p(x), _p(w_idx), L,
                                    _p(x_swa) if L else None, _p(swa) if L else None,
                                    _p(swa_pos) if L else None, _p(swa_len) if L else None)


# ------------------------------------------------ multi-query decode (next row)
def layer_group_multi(kv: KV, dm, n_rows, n_query: int, modes, q_idx, w, q, swa, swa_len, *,
                      top_k=512, pool_blocks=2048, sm_scale=None):
    """Q = n_query draft positions per sequence in one step.  Inputs carry a
    query axis after the batch axis (q_idx [L][B][Q][8][64], w [L][B][Q][8],
    q [L][B][Q][16][512]); the window is swa [L][B][128 + Q - 1][512] with
    swa_len [B].  Returns dict(idx [L][B][Q][k], idx_count [L][B][Q],
    pool [B][Q][pool_blocks], pool_count [B][Q], out [L][B][Q][16][512])."""
    n_rows = _c(n_rows, np.int64)
    modes = _c(modes, np.int32)
    q_idx = _c(q_idx, np.uint16)
    w = _c(w, np.float32)
    q = _c(q, np.uint16)
    swa = _c(swa, np.uint8)
    swa_len = _c(swa_len, np.int32)
    B, L, Q = len(n_rows), len(modes), int(n_query)
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(dm.d)
    idx = np.full((L, B, Q, top_k), -1, np.int32)
    idx_count = np.zeros((L, B, Q), np.int32)
    pb = max(pool_blocks, 1)
    pool_ = np.full((B, Q, pb), -1, np.int32)
    pool_count = np.zeros((B, Q), np.int32)
    out = np.zeros((L, B, Q, dm.h, dm.d), np.float64)
    rc = lib().csa2o_layer_group_multi(C.byref(kv.s), C.byref(dm), B, Q, _p(n_rows), L,
                                       _p(modes), _p(q_idx), _p(w), _p(q), _p(swa), _p(swa_len),
                                       top_k, pool_blocks, sm_scale, _p(idx), _p(idx_count),
                                       _p(pool_), _p(pool_count), _p(out))
    if rc:
        raise ValueError("oracle multi-query layer group: bad arguments or row outside the pool")
    return dict(idx=idx, idx_count=idx_count, pool=pool_[..., :pool_blocks],
                pool_count=pool_count, out=out)
