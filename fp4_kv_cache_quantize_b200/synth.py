"""Seeded synthetic inputs for the CSA2 decode step.

This module holds random draws and their storage formats only: it performs
none of the method's arithmetic (no FP4 packing, no scoring, no selection, no
attention).  Both the CUDA path and the CPU oracle take their inputs from here.

Every stream is numpy's Philox4x32-10 counter-based generator (Salmon et al.,
SC'11) keyed by (seed, stream id, chunk), so any chunk of any array can be
regenerated on its own, independent of thread count or of which other chunks
were drawn.  Storage conversions use library routines: float32 -> bf16 and
float32 -> E4M3 are torch's round-to-nearest-even casts.

Input recipe (shapes and distributions of the workloads):
  main KV x          bf16 [rows, 512], N(0,1) (optionally 0.1% of elements x50)
  indexer weights    bf16 [512, 64], N(0, 1/512)
  indexer K          bf16 [rows, 64] = bf16(x @ W_idx), fp64 sum of exact products
                     rounded once to bf16
  indexer query      bf16 [L, B, 8, 64], N(0,1)
  indexer head w     fp32 [L, B, 8], U(0,1)
  main query         bf16 [L, B, 16, 512], N(0,1)
  SWA window         E4M3 [L, B, 128, 512], N(0,1) cast to E4M3
Rows live in a row pool of 64-row pages; a sequence is either a contiguous run
of rows (seq_stride) or a page-table walk over a shuffled page pool.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

FULL, REINDEX, REUSE = 0, 1, 2
SEED_BASE = 0xC5A20000
CHUNK_ROWS = 4096
PAGE_ROWS = 64

# stream ids
_S_X, _S_OUT, _S_W, _S_QI, _S_WH, _S_Q, _S_SWA, _S_PLANT, _S_LEN, _S_PERM, _S_NOISE = range(11)


def rng(seed: int, stream: int, chunk: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=[int(seed) & 0xFFFFFFFFFFFFFFFF,
                                                     (stream << 40) | int(chunk)]))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def f64_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """bf16 bits of float64 values, rounded once to nearest-even (no float32
    step in between): 8 significant bits below the leading one, or the
    subnormal spacing 2^-133 below 2^-126."""
    x = np.asarray(a, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m 2^e, 0.5 <= |m| < 1
    e = np.maximum(e, -125)                 # bf16 subnormals: fixed spacing 2^-133
    r = np.ldexp(np.rint(np.ldexp(x, 8 - e)), e - 8)   # exact in float64; rint is RNE
    return to_bf16_bits(r.astype(np.float32))          # exact: r is a bf16 value


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def to_e4m3_bits(a: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


@dataclasses.dataclass
class Workload:
    """A seeded CSA2 decode workload (all host arrays, numpy)."""
    name: str
    seed: int
    B: int
    n_rows: np.ndarray          # int64 [B]   visible global entries C_b
    modes: np.ndarray           # int32 [L]
    pool_rows: int              # rows in the row pool
    seq_stride: int             # contiguous layout: row = b*seq_stride + p
    page_table: np.ndarray | None  # int32 [B, max_pages] or None
    top_k: int
    pool_blocks: int
    d: int = 512
    h: int = 16
    hi: int = 8
    di: int = 64
    blk: int = 8
    w: int = 128
    outlier_p: float = 0.0
    planted_blocks: int = 0
    planted_beta: float = 4.0
    # per-layer inputs (small)
    q_idx: np.ndarray | None = None   # uint16 [L, B, hi, di]
    w_h: np.ndarray | None = None     # float32 [L, B, hi]
    q: np.ndarray | None = None       # uint16 [L, B, h, d]
    swa: np.ndarray | None = None     # uint8  [L, B, w, d]
    swa_len: np.ndarray | None = None  # int32 [B]
    w_idx: np.ndarray | None = None   # uint16 [d, di]
    planted: np.ndarray | None = None  # int64 planted block ids of sequence 0

    @property
    def L(self) -> int:
        return len(self.modes)

    @property
    def n_chunks(self) -> int:
        return (self.pool_rows + CHUNK_ROWS - 1) // CHUNK_ROWS

    # ---- main KV rows -------------------------------------------------
    def x_chunk(self, c: int) -> np.ndarray:
        """bf16 bits of main-KV rows [c*CHUNK_ROWS, ...) of the row pool."""
        r0 = c * CHUNK_ROWS
        n = min(CHUNK_ROWS, self.pool_rows - r0)
        g = rng(self.seed, _S_X, c)
        x = g.standard_normal((n, self.d), dtype=np.float32)
        if self.outlier_p > 0:
            mask = rng(self.seed, _S_OUT, c).random((n, self.d), dtype=np.float32) < self.outlier_p
            x[mask] *= 50.0
        if self.planted is not None and len(self.planted):
            self._plant(x, r0)
        return to_bf16_bits(x)

    def _plant(self, x: np.ndarray, r0: int) -> None:
        # Planted high-similarity blocks of sequence 0 (contiguous layout):
        # rows of a planted block get beta * unit(W_idx u) added, where
        # u = sum_h w_h q_h of the first layer's indexer query.
        u = (self.w_h[0, 0][:, None].astype(np.float64) *
             bf16_bits_to_f32(self.q_idx[0, 0]).astype(np.float64)).sum(0)
        v = bf16_bits_to_f32(self.w_idx).astype(np.float64) @ u
        v /= np.linalg.norm(v)
        n = x.shape[0]
        for blk in self.planted:
            lo = int(blk) * self.blk - r0
            hi = lo + self.blk
            if hi <= 0 or lo >= n:
                continue
            x[max(lo, 0):min(hi, n)] += (self.planted_beta * v).astype(np.float32)

    def idxk_of(self, x_bits: np.ndarray) -> np.ndarray:
        """bf16 indexer K of bf16 main-KV rows: x @ W_idx summed in fp64 and
        rounded once to bf16 (nearest even), the cache-append rule."""
        xf = bf16_bits_to_f32(x_bits).astype(np.float64)
        wf = bf16_bits_to_f32(self.w_idx).astype(np.float64)
        return f64_to_bf16_bits(xf @ wf)

    def chunk(self, c: int):
        x = self.x_chunk(c)
        return x, self.idxk_of(x)

    def iter_chunks(self, threads: int | None = None):
        """Yield (row0, x_bits, idxk_bits) for every chunk, in order."""
        threads = threads or min(16, os.cpu_count() or 1)
        with ThreadPoolExecutor(threads) as ex:
            step = threads * 2
            for base in range(0, self.n_chunks, step):
                cs = list(range(base, min(base + step, self.n_chunks)))
                for c, (x, k) in zip(cs, ex.map(self.chunk, cs)):
                    yield c * CHUNK_ROWS, x, k

    def rows(self, rows: np.ndarray):
        """(x_bits, idxk_bits) of selected pool rows, regenerated chunk-wise."""
        rows = np.asarray(rows, dtype=np.int64)
        x = np.zeros((len(rows), self.d), np.uint16)
        k = np.zeros((len(rows), self.di), np.uint16)
        for c in np.unique(rows // CHUNK_ROWS):
            sel = np.nonzero(rows // CHUNK_ROWS == c)[0]
            xc, kc = self.chunk(int(c))
            x[sel] = xc[rows[sel] - c * CHUNK_ROWS]
            k[sel] = kc[rows[sel] - c * CHUNK_ROWS]
        return x, k

    def all_rows(self, threads: int | None = None):
        x = np.zeros((self.pool_rows, self.d), np.uint16)
        k = np.zeros((self.pool_rows, self.di), np.uint16)
        for r0, xc, kc in self.iter_chunks(threads):
            x[r0:r0 + len(xc)] = xc
            k[r0:r0 + len(kc)] = kc
        return x, k

    def row_of(self, b: int, p: np.ndarray) -> np.ndarray:
        p = np.asarray(p, dtype=np.int64)
        if self.page_table is None:
            return b * self.seq_stride + p
        return self.page_table[b, p // PAGE_ROWS].astype(np.int64) * PAGE_ROWS + p % PAGE_ROWS


def make(name: str, *, seed: int, B: int, n_rows, modes, top_k: int = 512,
         pool_blocks: int = 2048, paged: bool = False, outlier_p: float = 0.0,
         planted_blocks: int = 0, planted_beta: float = 4.0, swa_len=None,
         d: int = 512, h: int = 16, hi: int = 8, di: int = 64, blk: int = 8,
         w: int = 128) -> Workload:
    n_rows = np.asarray(n_rows, dtype=np.int64).reshape(B)
    modes = np.asarray(modes, dtype=np.int32)
    L = len(modes)
    if paged:
        pages = [(int(c) + PAGE_ROWS - 1) // PAGE_ROWS for c in n_rows]
        total = sum(pages)
        perm = rng(seed, _S_PERM).permutation(max(total, 1)).astype(np.int32)
        maxp = max(max(pages), 1)
        pt = np.zeros((B, maxp), np.int32)
        off = 0
        for b, n in enumerate(pages):
            pt[b, :n] = perm[off:off + n]
            off += n
        pool_rows = max(total, 1) * PAGE_ROWS
        seq_stride = 0
    else:
        pt = None
        seq_stride = int(max(int(n_rows.max()), 1))
        seq_stride = (seq_stride + PAGE_ROWS - 1) // PAGE_ROWS * PAGE_ROWS
        pool_rows = B * seq_stride
    wl = Workload(name=name, seed=seed, B=B, n_rows=n_rows, modes=modes,
                  pool_rows=pool_rows, seq_stride=seq_stride, page_table=pt,
                  top_k=top_k, pool_blocks=pool_blocks, d=d, h=h, hi=hi, di=di,
                  blk=blk, w=w, outlier_p=outlier_p, planted_blocks=planted_blocks,
                  planted_beta=planted_beta)
    wl.w_idx = to_bf16_bits(rng(seed, _S_W).standard_normal((d, di), dtype=np.float32)
                            / np.float32(np.sqrt(d)))
    wl.q_idx = to_bf16_bits(rng(seed, _S_QI).standard_normal((L, B, hi, di), dtype=np.float32))
    wl.w_h = rng(seed, _S_WH).random((L, B, hi), dtype=np.float32)
    wl.q = to_bf16_bits(rng(seed, _S_Q).standard_normal((L, B, h, d), dtype=np.float32))
    wl.swa = to_e4m3_bits(rng(seed, _S_SWA).standard_normal((L, B, w, d), dtype=np.float32))
    wl.swa_len = (np.full(B, w, np.int32) if swa_len is None
                  else np.asarray(swa_len, dtype=np.int32).reshape(B))
    if planted_blocks:
        nblk = (int(n_rows[0]) + blk - 1) // blk
        wl.planted = np.sort(rng(seed, _S_PLANT).choice(nblk, planted_blocks, replace=False))
        # Reindex layers: their indexer query is the first layer's plus N(0,1)
        # noise, so their picks overlap the Full layer's but differ.
        base = bf16_bits_to_f32(wl.q_idx[0])
        noise = rng(seed, _S_NOISE, 1 << 30).standard_normal(wl.q_idx.shape, dtype=np.float32)
        for l in range(1, L):
            if modes[l] == REINDEX:
                wl.q_idx[l] = to_bf16_bits(base + noise[l])
                wl.w_h[l] = wl.w_h[0]
    return wl


# --------------------------------------------------------------- presets
DECODER_20 = [FULL, REUSE, REUSE, REUSE] + [REINDEX, REUSE, REUSE, REUSE] * 4


def config(k: int) -> Workload:
    """The five benchmark workloads (0 tiny, 1 FP4 quantise, 2 HSI group,
    3 1M-context 20-layer decoder stack, 4 ragged paged batch)."""
    seed = SEED_BASE + k
    if k == 0:
        return make("tiny_4k_F3R", seed=seed, B=1, n_rows=[4096],
                    modes=[FULL, REUSE, REUSE, REUSE])
    if k == 1:
        return make("fp4_quant_1Mx512", seed=seed, B=1, n_rows=[1 << 20], modes=[],
                    outlier_p=0.001)
    if k == 2:
        return make("hsi_group_b8_128k", seed=seed, B=8, n_rows=[131072] * 8,
                    modes=[FULL, REINDEX, REUSE, REUSE, REUSE])
    if k == 3:
        return make("decoder20_1m", seed=seed, B=1, n_rows=[1 << 20], modes=DECODER_20,
                    planted_blocks=64)
    if k == 4:
        ctx = rng(seed, _S_LEN).integers(32768, 262144, size=64, endpoint=True)
        return make("ragged_paged_64seq_r2", seed=seed, B=64, n_rows=ctx // 2,
                    modes=[FULL] + [REUSE] * 5, pool_blocks=0, paged=True)
    raise ValueError(f"no workload {k}")
