"""Python binding of libcsa2.so (the C ABI declared in include/csa2.h).

Argument marshalling only: every function here takes torch tensors that live
on the current CUDA device, passes their pointers and the current stream to
the C entry point of the same name, and raises Csa2Error on a non-OK status.
All compute runs in the library's CUDA kernels.  There is no fallback: if
libcsa2.so is missing or fails to load, importing this module raises.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcsa2.so")

D, H, HI, DI, BLK, W = 512, 16, 8, 64, 8, 128
MAX_TOPK, MAX_POOL, MAX_ROWS = 512, 2048, 1 << 20
WS_HEADER = 256
FULL, REINDEX, REUSE = 0, 1, 2

STATUS = {0: "CSA2_OK", 1: "CSA2_ERR_INVALID_ARG", 2: "CSA2_ERR_SHAPE",
          3: "CSA2_ERR_ALIGNMENT", 4: "CSA2_ERR_WORKSPACE", 5: "CSA2_ERR_CUDA",
          6: "CSA2_ERR_TIMEOUT", 7: "CSA2_ERR_DEVICE_CHECK"}


class Csa2Error(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python -m fp4_kv_cache_quantize_b200.build`")
_lib = C.CDLL(LIB_PATH)


class KVView(C.Structure):
    _fields_ = [("codes", C.c_void_p), ("scales", C.c_void_p), ("idx_k", C.c_void_p),
                ("page_table", C.c_void_p), ("page_rows", C.c_int32),
                ("max_pages", C.c_int32), ("n_rows", C.c_void_p), ("batch", C.c_int32),
                ("max_rows", C.c_int32), ("seq_stride", C.c_int64), ("pool_rows", C.c_int64)]


class GroupDesc(C.Structure):
    _fields_ = [("kv", KVView), ("n_layers", C.c_int32), ("modes", C.c_void_p),
                ("q_idx", C.c_void_p), ("w", C.c_void_p), ("q", C.c_void_p),
                ("swa", C.c_void_p), ("swa_len", C.c_void_p), ("top_k", C.c_int32),
                ("pool_blocks", C.c_int32), ("sm_scale", C.c_float), ("idx", C.c_void_p),
                ("idx_count", C.c_void_p), ("pool", C.c_void_p), ("pool_count", C.c_void_p),
                ("out", C.c_void_p), ("n_query", C.c_int32)]


class TraceStruct(C.Structure):
    _fields_ = [("events", C.c_void_p * 64), ("names", C.c_char_p * 64),
                ("capacity", C.c_int32), ("count", C.c_int32)]


class _sig:
    """A C entry point, resolved from libcsa2.so on first call."""

    def __init__(self, name, restype, argtypes):
        self.name, self.restype, self.argtypes, self.f = name, restype, argtypes, None

    def __call__(self, *args):
        if self.f is None:
            f = getattr(_lib, self.name)
            f.restype, f.argtypes = self.restype, self.argtypes
            self.f = f
        return self.f(*args)


_vp, _i32, _i64, _sz = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t
_status_string = _sig("csa2_status_string", C.c_char_p, [C.c_int])
_last_error = _sig("csa2_last_error", C.c_char_p, [])
_workspace_init = _sig("csa2_workspace_init", C.c_int, [_vp, _sz, _vp])
_sync_status = _sig("csa2_sync_status", C.c_int, [_vp, _vp])
_quantize = _sig("csa2_quantize_fp4", C.c_int, [_vp, _i64, _i32, _vp, _vp, _vp])
_dequantize = _sig("csa2_dequantize_fp4", C.c_int, [_vp, _vp, _i64, _i32, _vp, _vp])
_index_ws = _sig("csa2_index_workspace_size", _sz, [C.POINTER(KVView), _i32, _i32])
_index_full = _sig("csa2_index_full", C.c_int,
                   [C.POINTER(KVView), _vp, _vp, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _sz, _vp])
_index_full_noalloc = _sig("csa2_index_full_noalloc", C.c_int,
                           [C.POINTER(KVView), _vp, _vp, _i32, _i32, _vp, _vp, _vp, _vp, _vp])
_index_reindex = _sig("csa2_index_reindex", C.c_int,
                      [C.POINTER(KVView), _vp, _vp, _vp, _vp, _i32, _i32, _vp, _vp, _vp, _sz,
                       _vp])
_attn_ws = _sig("csa2_attn_workspace_size", _sz, [_i32, _i32])
_attn = _sig("csa2_sparse_attn_decode", C.c_int,
             [_vp, C.POINTER(KVView), _vp, _vp, _i32, _vp, _vp, C.c_float, _vp, _vp, _sz, _vp])
_append = _sig("csa2_cache_append", C.c_int,
                [C.POINTER(KVView), _vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _sz, _vp])
_selftest_wait = _sig("csa2_selftest_bounded_wait", C.c_int, [_vp, _sz, _i64, _vp])
_trace_set = _sig("csa2_trace_set", None, [_vp])
_group_ws = _sig("csa2_group_workspace_size", _sz, [C.POINTER(GroupDesc)])
_group = _sig("csa2_layer_group", C.c_int, [C.POINTER(GroupDesc), _vp, _sz, _vp])


class CpShard(C.Structure):
    _fields_ = [("rank", C.c_int32), ("world", C.c_int32), ("shard_rows", C.c_int32)]


_PS = C.POINTER(CpShard)
_cp_ws = _sig("csa2_cp_workspace_size", _sz, [_PS, _i32, _i32, _i32])
_cp_partial_floats = _sig("csa2_cp_partial_floats", _sz, [_i32, _i32])
_cp_local_rows = _sig("csa2_cp_local_rows", C.c_int, [_PS, _vp, _i32, _vp, _vp, _sz, _vp])
_cp_block_max = _sig("csa2_cp_block_max", C.c_int,
                     [_PS, C.POINTER(KVView), _vp, _vp, _vp, _vp, _sz, _vp])
_cp_pool = _sig("csa2_cp_pool", C.c_int, [_PS, _vp, _vp, _i32, _i32, _vp, _vp, _vp, _sz, _vp])
_cp_filter = _sig("csa2_cp_filter", C.c_int,
                  [_PS, _i32, _vp, _vp, _i32, _i32, _vp, _vp, _i32, _vp, _vp, _vp, _sz, _vp])
_cp_select_local = _sig("csa2_cp_select_local", C.c_int,
                        [_PS, C.POINTER(KVView), _vp, _vp, _vp, _vp, _i32, _i32, _vp, _vp, _sz,
                         _vp])
_cp_select_merge = _sig("csa2_cp_select_merge", C.c_int,
                        [_PS, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _sz, _vp])
_cp_select_local_jobs = _sig("csa2_cp_select_local_jobs", C.c_int,
                             [_PS, C.POINTER(KVView), _i32, _vp, _i32, _vp, _vp, _vp, _vp, _i32,
                              _i32, _vp, _vp, _sz, _vp])
_cp_select_merge_jobs = _sig("csa2_cp_select_merge_jobs", C.c_int,
                             [_PS, _vp, _i32, _vp, _i32, _i32, _i32, _vp, _vp, _vp, _sz, _vp])
_cp_filter_layers = _sig("csa2_cp_filter_layers", C.c_int,
                         [_PS, _i32, _vp, _vp, _vp, _i32, _i32, _vp, _vp, _vp, _sz, _vp])
CP_MAX_JOBS = 8
_cp_attn_partial = _sig("csa2_cp_attn_partial", C.c_int,
                        [_PS, C.POINTER(KVView), _i32, _vp, _vp, _vp, _vp, _vp, _i32, C.c_float,
                         _vp, _vp, _sz, _vp])
_cp_attn_combine = _sig("csa2_cp_attn_combine", C.c_int,
                        [_PS, _vp, _i32, _i32, _vp, _vp, _sz, _vp])


def _check(rc: int):
    if rc != 0:
        raise Csa2Error(rc, _last_error().decode())


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on the CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def status_string(status: int) -> str:
    return _status_string(status).decode()


def last_error() -> str:
    return _last_error().decode()


# ------------------------------------------------------------------ views
class KVCache:
    """Device buffers of an FP4 main-KV cache and its indexer K, plus the row
    map (contiguous sequences or a page table).  Keeps its tensors alive."""

    def __init__(self, codes, scales, idx_k, n_rows, *, max_rows: int, seq_stride: int = 0,
                 page_table=None, page_rows: int = 64):
        self.codes, self.scales, self.idx_k = codes, scales, idx_k
        self.n_rows = n_rows.to(torch.int32).contiguous()
        self.page_table = None if page_table is None else page_table.to(torch.int32).contiguous()
        self.batch = int(self.n_rows.numel())
        self.view = KVView(_ptr(codes), _ptr(scales), _ptr(idx_k), _ptr(self.page_table),
                           page_rows, 0 if page_table is None else self.page_table.shape[1],
                           _ptr(self.n_rows), self.batch, int(max_rows), int(seq_stride),
                           int(codes.shape[0]))


def workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zero-initialised workspace of at least nbytes (16-byte aligned)."""
    ws = torch.zeros(max(int(nbytes), WS_HEADER), dtype=torch.uint8,
                     device=device or torch.cuda.current_device())
    return ws


# ------------------------------------------------------------- entry points
def csa2_workspace_init(ws, stream=None):
    _check(_workspace_init(_ptr(ws), ws.numel(), _stream(stream)))


def csa2_sync_status(ws, stream=None):
    _check(_sync_status(_ptr(ws), _stream(stream)))


def csa2_selftest_bounded_wait(ws, cycles: int, stream=None):
    _check(_selftest_wait(_ptr(ws), ws.numel(), int(cycles), _stream(stream)))


def csa2_quantize_fp4(x_bf16, codes, scales, stream=None):
    rows, ch = x_bf16.shape
    _check(_quantize(_ptr(x_bf16), rows, ch, _ptr(codes), _ptr(scales), _stream(stream)))


def csa2_dequantize_fp4(codes, scales, y_bf16, stream=None):
    rows, ch = y_bf16.shape
    _check(_dequantize(_ptr(codes), _ptr(scales), rows, ch, _ptr(y_bf16), _stream(stream)))


def csa2_index_workspace_size(kv: KVCache, top_k: int, pool_blocks: int) -> int:
    return _index_ws(C.byref(kv.view), top_k, pool_blocks)


def csa2_index_full(kv: KVCache, q_idx, w, top_k, pool_blocks, idx, idx_count, pool, pool_count,
                    ws, stream=None):
    _check(_index_full(C.byref(kv.view), _ptr(q_idx), _ptr(w), top_k, pool_blocks, _ptr(idx),
                       _ptr(idx_count), _ptr(pool), _ptr(pool_count), _ptr(ws), ws.numel(),
                       _stream(stream)))


def csa2_index_full_noalloc(kv: KVCache, q_idx, w, top_k, pool_blocks, idx, idx_count, pool,
                            pool_count, stream=None):
    """csa2_index_full with the library's static scratch instead of a
    caller workspace (for callers that cannot allocate device memory)."""
    _check(_index_full_noalloc(C.byref(kv.view), _ptr(q_idx), _ptr(w), top_k, pool_blocks,
                               _ptr(idx), _ptr(idx_count), _ptr(pool), _ptr(pool_count),
                               _stream(stream)))


def csa2_index_reindex(kv: KVCache, q_idx, w, pool, pool_count, pool_stride, top_k, idx,
                       idx_count, ws, stream=None):
    _check(_index_reindex(C.byref(kv.view), _ptr(q_idx), _ptr(w), _ptr(pool), _ptr(pool_count),
                          pool_stride, top_k, _ptr(idx), _ptr(idx_count), _ptr(ws), ws.numel(),
                          _stream(stream)))


def csa2_attn_workspace_size(batch: int, n_layers: int = 1) -> int:
    return _attn_ws(batch, n_layers)


def csa2_sparse_attn_decode(q, kv: KVCache, idx, idx_count, idx_stride, swa, swa_len, sm_scale,
                            out, ws, stream=None):
    _check(_attn(_ptr(q), C.byref(kv.view), _ptr(idx), _ptr(idx_count), idx_stride, _ptr(swa),
                 _ptr(swa_len), float(sm_scale), _ptr(out), _ptr(ws), ws.numel(),
                 _stream(stream)))


def csa2_cache_append(kv: KVCache, x, w_idx, ws, x_swa=None, swa=None, swa_pos=None,
                      swa_len=None, stream=None):
    """Append one step's entries: x bf16 [B][512] into the FP4 cache and its
    indexer K (w_idx bf16 [512][64]) at kv.n_rows (which advances), and
    x_swa bf16 [L][B][512] into the E4M3 window rings swa [L][B][128][512] at
    swa_pos % 128 (swa_pos advances, swa_len follows)."""
    L = 0 if x_swa is None else int(x_swa.shape[0])
    _check(_append(C.byref(kv.view), _ptr(x), _ptr(w_idx), L, _ptr(x_swa), _ptr(swa),
                   _ptr(swa_pos), _ptr(swa_len), _ptr(ws), ws.numel(), _stream(stream)))


class LayerGroup:
    """A csa2_group_desc over device tensors (kept alive by this object).
    With n_query = Q > 1 every per-query array has batch x Q rows (query axis
    after the batch axis) and swa holds 128 + Q - 1 rows per sequence."""

    def __init__(self, kv: KVCache, modes, q_idx, w, q, swa, swa_len, *, top_k=512,
                 pool_blocks=2048, sm_scale=None, idx=None, idx_count=None, pool=None,
                 pool_count=None, out=None, n_query=1):
        L, B = len(modes), kv.batch * max(int(n_query), 1)
        dev = q.device
        self.kv = kv
        self.modes_host = (C.c_int32 * L)(*[int(m) for m in modes])
        self.q_idx, self.w, self.q, self.swa = q_idx, w, q, swa
        self.swa_len = swa_len.to(torch.int32).contiguous()
        self.idx = idx if idx is not None else torch.empty((L, B, top_k), dtype=torch.int32,
                                                           device=dev)
        self.idx_count = idx_count if idx_count is not None else torch.empty(
            (L, B), dtype=torch.int32, device=dev)
        pb = max(pool_blocks, 1)
        self.pool = pool if pool is not None else torch.empty((B, pb), dtype=torch.int32,
                                                              device=dev)
        self.pool_count = pool_count if pool_count is not None else torch.empty(
            (B,), dtype=torch.int32, device=dev)
        self.out = out if out is not None else torch.empty((L, B, H, D), dtype=torch.bfloat16,
                                                           device=dev)
        if sm_scale is None:
            sm_scale = D ** -0.5
        self.desc = GroupDesc(kv.view, L, C.cast(self.modes_host, C.c_void_p).value, _ptr(q_idx),
                              _ptr(w), _ptr(q), _ptr(swa), _ptr(self.swa_len), top_k,
                              pool_blocks, float(sm_scale), _ptr(self.idx),
                              _ptr(self.idx_count), _ptr(self.pool), _ptr(self.pool_count),
                              _ptr(self.out), int(n_query))

    def workspace_size(self) -> int:
        return _group_ws(C.byref(self.desc))


def csa2_group_workspace_size(group: LayerGroup) -> int:
    return group.workspace_size()


def csa2_layer_group(group: LayerGroup, ws, stream=None):
    _check(_group(C.byref(group.desc), _ptr(ws), ws.numel(), _stream(stream)))


class Trace:
    """Per-launch event trace (csa2_trace).  events: torch.cuda.Event objects
    created with enable_timing=True and already recorded once (so that their
    CUDA events exist)."""

    def __init__(self, events):
        self.events = list(events)[:64]
        self.s = TraceStruct()
        for i, e in enumerate(self.events):
            self.s.events[i] = e.cuda_event
        self.s.capacity = len(self.events)
        self.s.count = 0

    def names(self):
        return [self.s.names[i].decode() for i in range(self.s.count)]


def csa2_trace_set(trace):
    _trace_set(C.addressof(trace.s) if trace is not None else None)


# ------------------------------------------------- context-parallel decode
def csa2_cp_workspace_size(shard: CpShard, batch: int, n_layers: int, top_k: int) -> int:
    return _cp_ws(C.byref(shard), batch, n_layers, top_k)


def csa2_cp_partial_floats(batch: int, n_layers: int) -> int:
    return _cp_partial_floats(batch, n_layers)


def csa2_cp_local_rows(shard: CpShard, n_rows, local_rows, ws, stream=None):
    _check(_cp_local_rows(C.byref(shard), _ptr(n_rows), int(n_rows.numel()), _ptr(local_rows),
                          _ptr(ws), ws.numel(), _stream(stream)))


def csa2_cp_block_max(shard: CpShard, kv: KVCache, q_idx, w, bm, ws, stream=None):
    _check(_cp_block_max(C.byref(shard), C.byref(kv.view), _ptr(q_idx), _ptr(w), _ptr(bm),
                         _ptr(ws), ws.numel(), _stream(stream)))


def csa2_cp_pool(shard: CpShard, bm_all, n_rows, P, pool, pool_count, ws, stream=None):
    _check(_cp_pool(C.byref(shard), _ptr(bm_all), _ptr(n_rows), int(n_rows.numel()), P,
                    _ptr(pool), _ptr(pool_count), _ptr(ws), ws.numel(), _stream(stream)))


def csa2_cp_filter(shard: CpShard, unit, lst, count, out, out_count, ws, copy=None,
                   copy_count=None, stream=None):
    """lst int32 [batch][stride] -> out int32 [batch][out_stride] (see csa2.h)."""
    _check(_cp_filter(C.byref(shard), unit, _ptr(lst), _ptr(count), int(lst.shape[-1]),
                      int(count.numel()), _ptr(out), _ptr(out_count), int(out.shape[-1]),
                      _ptr(copy), _ptr(copy_count), _ptr(ws), ws.numel(),
                      _stream(stream)))


def csa2_cp_select_local(shard: CpShard, kv: KVCache, q_idx, w, cand, cand_count, top_k, send,
                         ws, stream=None):
    _check(_cp_select_local(C.byref(shard), C.byref(kv.view), _ptr(q_idx), _ptr(w),
                            _ptr(cand), _ptr(cand_count), int(cand.shape[-1]), top_k,
                            _ptr(send), _ptr(ws), ws.numel(), _stream(stream)))


def csa2_cp_select_merge(shard: CpShard, gathered, n_jobs, job, batch, top_k, idx, idx_count,
                         ws, stream=None):
    _check(_cp_select_merge(C.byref(shard), _ptr(gathered), n_jobs, job, batch, top_k,
                            _ptr(idx), _ptr(idx_count), _ptr(ws), ws.numel(),
                            _stream(stream)))


def _host_i32(values):
    arr = (C.c_int32 * len(values))(*[int(v) for v in values])
    return arr


def csa2_cp_select_local_jobs(shard: CpShard, kv: KVCache, layers, q_idx, w, cand, cand_count,
                              top_k, send, ws, stream=None):
    """Jobs = layers (host list) of q_idx [L][B][8][64] / w [L][B][8]; send
    [J][B][top_k][2] (see csa2.h)."""
    arr = _host_i32(layers)
    _check(_cp_select_local_jobs(C.byref(shard), C.byref(kv.view), len(layers), arr,
                                 int(q_idx.shape[0]), _ptr(q_idx), _ptr(w), _ptr(cand),
                                 _ptr(cand_count), int(cand.shape[-1]), top_k, _ptr(send),
                                 _ptr(ws), ws.numel(), _stream(stream)))


def csa2_cp_select_merge_jobs(shard: CpShard, gathered, layers, batch, top_k, idx, idx_count,
                              ws, stream=None):
    """Jobs 0..J-1 of gathered -> layers (host list) of idx [L][B][top_k]."""
    arr = _host_i32(layers)
    _check(_cp_select_merge_jobs(C.byref(shard), _ptr(gathered), len(layers), arr,
                                 int(idx.shape[0]), batch, top_k, _ptr(idx), _ptr(idx_count),
                                 _ptr(ws), ws.numel(), _stream(stream)))


def csa2_cp_filter_layers(shard: CpShard, src, idx, idx_count, idx_local, idx_local_count, ws,
                          stream=None):
    """Every layer's rows this shard owns: idx [L][B][K] -> idx_local (src:
    host list of the layer each layer reads; see csa2.h)."""
    arr = _host_i32(src)
    _check(_cp_filter_layers(C.byref(shard), len(src), arr, _ptr(idx), _ptr(idx_count),
                             int(idx.shape[-1]), int(idx.shape[1]), _ptr(idx_local),
                             _ptr(idx_local_count), _ptr(ws), ws.numel(), _stream(stream)))


def csa2_cp_attn_partial(shard: CpShard, kv: KVCache, q, swa, swa_len, idx_local, idx_count,
                         sm_scale, partial, ws, stream=None):
    L = int(q.shape[0])
    _check(_cp_attn_partial(C.byref(shard), C.byref(kv.view), L, _ptr(q), _ptr(swa),
                            _ptr(swa_len), _ptr(idx_local), _ptr(idx_count),
                            int(idx_local.shape[-1]), float(sm_scale), _ptr(partial), _ptr(ws),
                            ws.numel(), _stream(stream)))


def csa2_cp_attn_combine(shard: CpShard, gathered, n_layers, batch, out, ws, stream=None):
    _check(_cp_attn_combine(C.byref(shard), _ptr(gathered), n_layers, batch, _ptr(out),
                            _ptr(ws), ws.numel(), _stream(stream)))
