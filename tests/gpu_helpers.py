"""Helpers of the GPU parity tests: move seeded workloads to the device, run
the C ABI, and compare with the CPU oracle under the stated tolerances.

Tolerances:
  * FP4 codes and scales: bit-exact.
  * Selected index sets: exact, except positions whose oracle score lies within
    1e-5 (relative) of the oracle's k-th score; a pool block may differ only
    when its oracle block maximum lies within 1e-5 of the pool threshold.
  * Attention outputs: relative L2 error <= 5e-3 per (layer, sequence).
"""
from __future__ import annotations

import numpy as np
import torch

from fp4_kv_cache_quantize_b200 import synth

SEL_RTOL = 1e-5
ATTN_RTOL = 5e-3


def dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16))
    else:
        t = torch.from_numpy(a)
    t = t.cuda()
    return t.view(dtype) if dtype is not None else t


class DeviceWorkload:
    """A synth.Workload on the GPU: FP4 cache, indexer K, per-layer inputs."""

    def __init__(self, lib, wl: synth.Workload, orc=None, oracle_codes: bool = True):
        self.wl = wl
        rows = wl.pool_rows
        if oracle_codes:
            # small workloads: the oracle quantises, both sides read its bytes
            x, k = wl.all_rows()
            self.codes_np, self.scales_np = orc.quantize_fp4(x)
            self.idxk_np = k
            self.codes, self.scales = dev(self.codes_np), dev(self.scales_np)
            self.idxk = dev(k)
        else:
            # large workloads: quantised on the GPU (bit-exactness of the pack
            # kernel is tested on its own); the oracle regenerates what it needs
            self.codes = torch.empty((rows, 256), dtype=torch.uint8, device="cuda")
            self.scales = torch.empty((rows, 32), dtype=torch.uint8, device="cuda")
            self.idxk = torch.empty((rows, 64), dtype=torch.int16, device="cuda")
            self.idxk_np = np.zeros((rows, 64), np.uint16)
            for r0, xc, kc in wl.iter_chunks():
                n = len(xc)
                xd = dev(xc)
                lib.csa2_quantize_fp4(xd.view(torch.bfloat16), self.codes[r0:r0 + n],
                                      self.scales[r0:r0 + n])
                self.idxk[r0:r0 + n] = dev(kc)
                self.idxk_np[r0:r0 + n] = kc
            self.codes_np = self.scales_np = None
        self.n_rows = dev(wl.n_rows.astype(np.int32))
        self.page_table = None if wl.page_table is None else dev(wl.page_table)
        self.kv = lib.KVCache(self.codes, self.scales, self.idxk, self.n_rows,
                              max_rows=int(wl.n_rows.max()), seq_stride=wl.seq_stride,
                              page_table=self.page_table)
        self.q_idx = dev(wl.q_idx)
        self.w = dev(wl.w_h)
        self.q = dev(wl.q)
        self.swa = dev(wl.swa)
        self.swa_len = dev(wl.swa_len)

    def oracle_kv(self, orc):
        return orc.KV(self.codes_np, self.scales_np, self.idxk_np, seq_stride=self.wl.seq_stride,
                      page_table=self.wl.page_table)


def kth_threshold(scores: np.ndarray, k: int) -> float:
    k = min(k, len(scores))
    return float(np.sort(scores)[::-1][k - 1]) if k > 0 else 0.0


def check_selection(gpu_idx: np.ndarray, gpu_cnt: int, want_idx: np.ndarray,
                    score_of, k: int, cand_positions: np.ndarray | None = None,
                    extra_ok=None, what=""):
    """gpu_idx: the GPU's selection (ascending, -1 padded); want_idx: the
    oracle's; score_of(positions) -> oracle fp64 scores."""
    assert gpu_cnt == len(want_idx), f"{what}: count {gpu_cnt} != {len(want_idx)}"
    g = gpu_idx[:gpu_cnt]
    assert np.all(gpu_idx[gpu_cnt:] == -1), f"{what}: padding not -1"
    assert np.all(np.diff(g) > 0), f"{what}: not strictly ascending"
    diff = np.setxor1d(g, want_idx)
    if len(diff) == 0:
        return 0
    cand = cand_positions if cand_positions is not None else None
    s_all = score_of(cand) if cand is not None else None
    thr = kth_threshold(s_all, k) if s_all is not None else float(np.min(score_of(want_idx)))
    s = score_of(diff)
    near = np.abs(s - thr) <= SEL_RTOL * max(abs(thr), 1e-30)
    if extra_ok is not None:
        near |= extra_ok(diff)
    assert np.all(near), (f"{what}: {int((~near).sum())} positions differ beyond the tie "
                          f"tolerance; e.g. {diff[~near][:5]} scores {s[~near][:5]} thr {thr}")
    return len(diff)


def rel_l2(got: np.ndarray, want: np.ndarray) -> float:
    den = np.linalg.norm(want)
    return float(np.linalg.norm(got - want) / (den if den > 0 else 1.0))


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)
