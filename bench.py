"""Benchmark of the CSA2 decode step over an FP4 global KV cache.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl csa2|reference]
                    [--config 3]

One step = one decode step of a whole CSA2 layer group (csa2_layer_group):
Full-layer indexer scan + HSI pool + Top-512, Reindex rescoring, Reuse, and
sparse + SWA attention of every layer.  The default workload is the 1M-context
20-layer decoder stack (batch 1, context 1,048,576, [F,R,R,R] + 4 x [X,R,R,R],
64 planted blocks).  Metric: decode layer-steps/s (batch x layers / step time).

Timing: CUDA events on the launching stream around every step, L2 flushed
(256 MiB write) between steps outside the events, W warm-up steps, max over
ranks.  --gpus N > 1 runs N independent replicas (the decode step has no
exchange to make across GPUs), one per rank, launched by torchrun.
The reference arm (--impl reference) times the CPU oracle on the host cores.

Beside the headline step the line carries, under "next_rows", the cache-append
call, a 4-query (draft verification) step, a 64-token prefill chunk, and the
context-parallel step with every sequence cut into 8 shards run on this one
GPU (checked against the one-device step's indices, pool and output).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA2 decode layer-steps/s and achieved HBM GB/s vs 8 TB/s at 128K–1M ctx"
UNIT = "layer-steps/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
ATTN_BYTES = 512 * 288 + 128 * 512 + 2 * 16384 + 2048   # per layer per sequence


def algorithmic_bytes(wl) -> dict:
    """Bytes the method must move per step (intermediates excluded)."""
    C = wl.n_rows.astype(np.int64)
    full = int(sum(128 * int(c) for c in C)) * int((wl.modes == 0).sum())
    pool_pos = min(wl.pool_blocks, 1 << 30) * 8 if wl.pool_blocks else None
    rx = 0
    for _ in range(int((wl.modes == 1).sum())):
        rx += int(sum(128 * (min(pool_pos, int(c)) if pool_pos else int(c)) for c in C))
    attn = ATTN_BYTES * wl.B * wl.L
    return {"scan": full, "reindex": rx, "attn": attn, "total": full + rx + attn}


def measured_peaks() -> tuple[float, str]:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            return float(json.load(fh)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def profile_value(name, key):
    """An integer recorded as `key: value` in a committed ncu summary."""
    try:
        with open(os.path.join(ROOT, "profiles", name)) as fh:
            for line in fh:
                if line.startswith(key + ":"):
                    return int(line.split(":", 1)[1].strip().split()[0])
    except OSError:
        pass
    return None


def scan_traffic_from_profile():
    """dram bytes per scan launch from the committed ncu summary, if any."""
    path = os.path.join(ROOT, "profiles", "scan_decoder20_1m.md")
    try:
        with open(path) as fh:
            for line in fh:
                if line.startswith("dram_bytes_per_launch:"):
                    return int(line.split(":", 1)[1].strip().split()[0])
    except OSError:
        pass
    return None


class ClockSampler:
    """NVML sampling of SM clock and throttle reasons while running."""

    def __init__(self, index: int):
        self.samples, self.reasons, self.ok = [], set(), False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        nv = self.nv
        names = {
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for k, bit in names.items():
                    if r & bit:
                        self.reasons.add(k)
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------ ranks
def max_over_ranks(x: float, dist=None, device=None) -> float:
    """The largest x over all ranks (device time of the slowest replica)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, t_ms: float) -> float:
    """Whole-job units per second: every rank's units over the slowest time."""
    return units_per_rank * world / (t_ms * 1e-3)


# ------------------------------------------------------------ oracle (CPU)
def oracle_step_setup(wl):
    """The CPU oracle's inputs for one step of this workload.

    The oracle reads main-KV codes only at the rows it selects, so a first
    (untimed) pass with zero codes finds those rows, and the oracle quantises
    them from the seeded bf16 rows; the timed passes run on the real bytes."""
    import oracle

    dm = oracle.dims()
    rows_needed = set()
    codes = np.zeros((wl.pool_rows, 256), np.uint8)
    scales = np.zeros((wl.pool_rows, 32), np.uint8)
    idxk = np.zeros((wl.pool_rows, 64), np.uint16)
    for r0, _, kc in wl.iter_chunks():
        idxk[r0:r0 + len(kc)] = kc
    kv = oracle.KV(codes, scales, idxk, seq_stride=wl.seq_stride, page_table=wl.page_table)
    r = oracle.layer_group(kv, dm, wl.n_rows, wl.modes, wl.q_idx, wl.w_h, wl.q, wl.swa,
                           wl.swa_len, top_k=wl.top_k, pool_blocks=wl.pool_blocks)
    for l in range(wl.L):
        for b in range(wl.B):
            pos = r["idx"][l, b, :r["idx_count"][l, b]]
            rows_needed.update(wl.row_of(b, pos).tolist())
    x_sel_rows = np.array(sorted(rows_needed), dtype=np.int64)
    xs, _ = wl.rows(x_sel_rows)
    c, s_ = oracle.quantize_fp4(xs)
    kv.codes[x_sel_rows] = c
    kv.scales[x_sel_rows] = s_

    def step():
        t0 = time.perf_counter()
        oracle.layer_group(kv, dm, wl.n_rows, wl.modes, wl.q_idx, wl.w_h, wl.q, wl.swa,
                           wl.swa_len, top_k=wl.top_k, pool_blocks=wl.pool_blocks)
        return time.perf_counter() - t0
    return step


def oracle_step_time(wl):
    """One full step of the CPU oracle on this workload, in seconds."""
    return oracle_step_setup(wl)()


REFERENCE_BUDGET_S = 150.0


def reference_counts(warmup, steps, t_step, budget_s=REFERENCE_BUDGET_S):
    """(warm-up steps, timed steps) of the reference arm: the requested counts,
    or as many as fit the budget at t_step seconds a step (at least one of
    each; warm-ups take at most a tenth of the budget)."""
    fit = max(1, int(budget_s / max(t_step, 1e-6)))
    warm = max(1, min(warmup, max(1, fit // 10)))
    timed = max(1, min(steps, fit - warm))
    return warm, timed


def run_reference(args, wl, rank):
    """The oracle as the reference arm: W warm-up and K timed full steps on one
    host core, as many of each as fit the time budget (a full 1M-context step
    takes seconds in fp64 C); the line states the counts it ran."""
    if rank != 0:
        return
    step = oracle_step_setup(wl)
    t_first = step()                     # the first warm-up step
    warm, timed = reference_counts(args.warmup, args.steps, t_first)
    for _ in range(warm - 1):
        step()
    dts = [step() for _ in range(timed)]
    dt = sum(dts) / len(dts)
    value = wl.B * wl.L / dt
    sample = (f"{timed} full decode steps of {wl.name} after {warm} warm-up steps "
              f"({args.steps} and {args.warmup} requested; as many as fit "
              f"{REFERENCE_BUDGET_S:.0f} s), single-threaded C, fp64, full-sort selection")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": timed, "warmup": warm, "ms_per_step": dt * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_dict(wl),
            "cpu_baseline": {"kind": "oracle", "value": value, "unit": UNIT, "cores": 1,
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_dict(wl):
    return {"workload": wl.name, "batch": int(wl.B), "context": int(wl.n_rows.max()),
            "layers": int(wl.L), "modes": "".join("FXR"[m] for m in wl.modes),
            "top_k": int(wl.top_k), "pool_blocks": int(wl.pool_blocks),
            "l2": "flushed between timed steps: 256 MiB written then 256 MiB read"}


# ------------------------------------------------------------ GPU arm
def time_cache_append(csa2, wl, dev, stream, K, W, with_cpu):
    """The cache-append step that precedes a decode step (one new main-KV
    entry per sequence, one window entry per layer and sequence), timed with
    events over K back-to-back calls into a scratch cache of the workload's
    batch and layer count.  Latency-bound: it moves ~100 KB per call.  The
    oracle's append is timed on the same inputs (host copies)."""
    import torch
    from fp4_kv_cache_quantize_b200 import synth
    B, L = wl.B, wl.L
    cap = 64 * ((W + K + 63) // 64 + 1)
    rng = synth.rng(wl.seed, 200)
    x_np = synth.to_bf16_bits(rng.standard_normal((B, 512)).astype(np.float32))
    w_np = synth.to_bf16_bits((rng.standard_normal((512, 64)) / 512 ** 0.5).astype(np.float32))
    xs_np = synth.to_bf16_bits(rng.standard_normal((L, B, 512)).astype(np.float32))
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev)  # noqa: E731
    codes = torch.zeros((B * cap, 256), dtype=torch.uint8, device=dev)
    scales = torch.zeros((B * cap, 32), dtype=torch.uint8, device=dev)
    idxk = torch.zeros((B * cap, 64), dtype=torch.int16, device=dev)
    n_rows = torch.zeros(B, dtype=torch.int32, device=dev)
    kv = csa2.KVCache(codes, scales, idxk, n_rows, max_rows=cap, seq_stride=cap)
    x, w_idx, x_swa = to_dev(x_np), to_dev(w_np), to_dev(xs_np)
    swa = torch.zeros((L, B, 128, 512), dtype=torch.uint8, device=dev)
    swa_pos = torch.zeros(B, dtype=torch.int32, device=dev)
    swa_len = torch.zeros(B, dtype=torch.int32, device=dev)
    ws = csa2.workspace(csa2.WS_HEADER, device=dev)

    def call():
        csa2.csa2_cache_append(kv, x, w_idx, ws, x_swa, swa, swa_pos, swa_len)

    for _ in range(W):
        call()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(K):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    csa2.csa2_sync_status(ws)
    assert int(n_rows.min()) == W + K and int(swa_pos.min()) == W + K
    us = 1e3 * e0.elapsed_time(e1) / K
    per_seq = 1024 + 256 + 32 + 128 + L * (1024 + 512)
    nbytes = B * per_seq + 512 * 64 * 2
    peak, peak_kind = measured_peaks()
    out = {"us_per_call": us, "launches_per_call": 2, "batch": B, "layers": L,
           "algorithmic_bytes_per_call": nbytes,
           "roofline": {"bound": "latency", "achieved": nbytes / (us * 1e-6) / 1e9, "peak": peak,
                        "peak_kind": peak_kind, "unit": "GB/s",
                        "frac": nbytes / (us * 1e-6) / 1e9 / peak, "traffic": None},
           "timing": f"{K} back-to-back calls after {W} warm-up calls, CUDA events"}
    if with_cpu:
        import oracle
        dm = oracle.dims()
        okv = oracle.KV(np.zeros((B * cap, 256), np.uint8), np.zeros((B * cap, 32), np.uint8),
                        np.zeros((B * cap, 64), np.uint16), seq_stride=cap)
        on = np.zeros(B, np.int64)
        oswa = np.zeros((L, B, 128, 512), np.uint8)
        opos, olen = np.zeros(B, np.int64), np.zeros(B, np.int32)
        n_calls = 20
        t0 = time.perf_counter()
        for _ in range(n_calls):
            oracle.cache_append(okv, dm, on, x_np, w_np, xs_np, oswa, opos, olen)
        dt = (time.perf_counter() - t0) / n_calls
        out["cpu_baseline"] = {"value": dt * 1e6, "unit": "us_per_call", "cores": 1,
                               "kind": "oracle",
                               "sample": f"{n_calls} oracle appends of the same inputs"}
    return out


def oracle_multi_time(wl, Q, q_idx, w, q, swa, swa_len):
    """The oracle's multi-query step on this workload (one step), with the
    main-KV rows it reads quantised as in oracle_step_time."""
    import oracle
    dm = oracle.dims()
    codes = np.zeros((wl.pool_rows, 256), np.uint8)
    scales = np.zeros((wl.pool_rows, 32), np.uint8)
    idxk = np.zeros((wl.pool_rows, 64), np.uint16)
    for r0, _, kc in wl.iter_chunks():
        idxk[r0:r0 + len(kc)] = kc
    kv = oracle.KV(codes, scales, idxk, seq_stride=wl.seq_stride, page_table=wl.page_table)
    args = (kv, dm, wl.n_rows, Q, wl.modes, q_idx, w, q, swa, swa_len)
    r = oracle.layer_group_multi(*args, top_k=wl.top_k, pool_blocks=wl.pool_blocks)
    rows = set()
    for b in range(wl.B):
        for t in range(Q):
            for l in range(wl.L):
                pos = r["idx"][l, b, t, :r["idx_count"][l, b, t]]
                rows.update(wl.row_of(b, pos).tolist())
    sel = np.array(sorted(rows), dtype=np.int64)
    xs, _ = wl.rows(sel)
    c, sc = oracle.quantize_fp4(xs)
    kv.codes[sel] = c
    kv.scales[sel] = sc
    t0 = time.perf_counter()
    oracle.layer_group_multi(*args, top_k=wl.top_k, pool_blocks=wl.pool_blocks)
    return time.perf_counter() - t0


def time_multi_query(csa2, wl, kv, dev, stream, flush_l2, K, W, with_cpu, Q=4):
    """Verification of Q draft positions per sequence in one step over the
    workload's cache (the last Q entries are the drafts), timed like the
    headline step (L2 flushed between steps, events around each step), plus
    a traced pass for the scan's roofline and the oracle beside it."""
    import torch
    from fp4_kv_cache_quantize_b200 import synth
    B, L = wl.B, wl.L
    rng = synth.rng(wl.seed, 300 + Q)
    bf = lambda *shape: synth.to_bf16_bits(rng.standard_normal(shape).astype(np.float32))  # noqa: E731
    q_idx_np, q_np = bf(L, B, Q, 8, 64), bf(L, B, Q, 16, 512)
    w_np = rng.uniform(0, 1, (L, B, Q, 8)).astype(np.float32)
    swa_np = synth.to_e4m3_bits(rng.standard_normal((L, B, 128 + Q - 1, 512)).astype(np.float32))
    swa_len_np = np.full(B, 128 + Q - 1, np.int32)
    to_dev = lambda a: torch.from_numpy(np.ascontiguousarray(  # noqa: E731
        a.view(np.int16) if a.dtype == np.uint16 else a)).to(dev)
    grp = csa2.LayerGroup(kv, wl.modes, to_dev(q_idx_np.reshape(L, B * Q, 8, 64)),
                          to_dev(w_np.reshape(L, B * Q, 8)), to_dev(q_np.reshape(L, B * Q, 16, 512)),
                          to_dev(swa_np), to_dev(swa_len_np), top_k=wl.top_k,
                          pool_blocks=wl.pool_blocks, n_query=Q)
    ws = csa2.workspace(grp.workspace_size(), device=dev)
    for _ in range(W):
        csa2.csa2_layer_group(grp, ws)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    torch.cuda.synchronize()
    for i in range(K):
        flush_l2()
        ev[i][0].record(stream)
        csa2.csa2_layer_group(grp, ws)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    csa2.csa2_sync_status(ws)
    ms = sum(a.elapsed_time(b) for a, b in ev) / K
    # traced pass: the scan's own duration for its roofline
    n_ev, KT = 32, min(K, 20)
    tev = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev * KT)]
    for e in tev:
        e.record(stream)
    torch.cuda.synchronize()
    scan_ms = []
    for i in range(KT):
        tr = csa2.Trace(tev[i * n_ev:(i + 1) * n_ev])
        flush_l2()
        csa2.csa2_trace_set(tr)
        csa2.csa2_layer_group(grp, ws)
        csa2.csa2_trace_set(None)
        torch.cuda.synchronize()
        names = tr.names()
        for j in range(len(names) - 1):
            if names[j] == "scan":
                scan_ms.append(tr.events[j].elapsed_time(tr.events[j + 1]))
    scan_bytes = 128 * int(wl.n_rows.sum())
    peak, peak_kind = measured_peaks()
    t_scan = sum(scan_ms) / len(scan_ms) * 1e-3
    out = {"queries_per_sequence": Q, "ms_per_step": ms,
           "value": B * Q * L / (ms * 1e-3), "unit": "query-layer-steps/s",
           "steps": K, "warmup": W,
           "roofline": {"bound": "hbm", "kernel": "score_scan_kernel (N = 8Q)",
                        "achieved": scan_bytes / t_scan / 1e9, "peak": peak,
                        "peak_kind": peak_kind, "unit": "GB/s",
                        "frac": scan_bytes / t_scan / 1e9 / peak, "traffic": None,
                        "algorithmic_bytes_per_launch": scan_bytes},
           "note": "indexer K read once per step for all queries (MMA N = 8Q)"}
    if with_cpu:
        # a bounded sample: the last S queries, which see exactly what they see
        # as part of all Q (the window slice keeps their rows)
        S = min(Q, 4)
        dt = oracle_multi_time(wl, S, np.ascontiguousarray(q_idx_np[:, :, Q - S:]),
                               np.ascontiguousarray(w_np[:, :, Q - S:]),
                               np.ascontiguousarray(q_np[:, :, Q - S:]),
                               np.ascontiguousarray(swa_np[:, :, Q - S:]), swa_len_np - (Q - S))
        out["cpu_baseline"] = {"value": B * S * L / dt, "unit": "query-layer-steps/s",
                               "cores": 1, "kind": "oracle",
                               "sample": (f"the last {S} of the {Q} queries of one step of "
                                          f"{wl.name}, one host core")}
    return out


def time_layer_sequential(csa2, wl, kv, bufs, grp, stream, flush_l2, K, W):
    """The same layer group as a layer-sequential schedule: each layer's index
    step (csa2_index_full / csa2_index_reindex) and attention
    (csa2_sparse_attn_decode) run after the previous layer's, as a decoder whose
    queries come from the previous layer would run them.  Timed like the
    headline (one CUDA graph per step when capture works, L2 flushed between
    steps); its indices must equal the grouped step's."""
    import torch
    q_idx, w_h, q, swa, swa_len = bufs
    dev = q.device
    L, B, Kk, P = wl.L, wl.B, wl.top_k, wl.pool_blocks
    modes = [int(m) for m in wl.modes]
    i32 = dict(dtype=torch.int32, device=dev)
    idx = torch.full((L, B, Kk), -1, **i32)
    # per-layer counts on 16-byte boundaries (the entry points' alignment rule)
    cnt_rows = torch.zeros((L, (B + 3) // 4 * 4), **i32)
    cnt = [cnt_rows[l, :B] for l in range(L)]
    pool = torch.full((B, max(P, 1)), -1, **i32)
    pcnt = torch.zeros((B,), **i32)
    out = torch.zeros((L, B, 16, 512), dtype=torch.bfloat16, device=dev)
    ws_i = csa2.workspace(csa2.csa2_index_workspace_size(kv, Kk, P), device=dev)
    ws_a = csa2.workspace(csa2.csa2_attn_workspace_size(B, 1), device=dev)
    sm = csa2.D ** -0.5

    def step():
        src = 0
        for l, m in enumerate(modes):
            if m == 0:
                csa2.csa2_index_full(kv, q_idx[l], w_h[l], Kk, P, idx[l], cnt[l],
                                     pool if P else None, pcnt if P else None, ws_i)
                src = l
            elif m == 1:
                csa2.csa2_index_reindex(kv, q_idx[l], w_h[l], pool if P else None,
                                        pcnt if P else None, max(P, 1), Kk, idx[l], cnt[l], ws_i)
                src = l
            csa2.csa2_sparse_attn_decode(q[l], kv, idx[src], cnt[src], Kk, swa[l], swa_len, sm,
                                         out[l], ws_a)

    for _ in range(W):
        step()
    torch.cuda.synchronize()
    csa2.csa2_sync_status(ws_i)
    csa2.csa2_sync_status(ws_a)
    # REUSE layers of the grouped step hold copies of their source's indices
    src_of, src = [], 0
    for l, m in enumerate(modes):
        src = l if m != 2 else src
        src_of.append(src)
    same = all(torch.equal(idx[src_of[l]], grp.idx[l]) and torch.equal(cnt[src_of[l]],
                                                                        grp.idx_count[l])
               for l in range(L))
    a, b = out.double(), grp.out.double()
    err = float((a - b).norm() / max(float(b.norm()), 1e-30))

    def timed(run):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]
        for i in range(K):
            flush_l2()
            ev[i][0].record(stream)
            run()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        return sorted(x.elapsed_time(y) for x, y in ev)

    launch, times = "direct", None
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        torch.cuda.synchronize()
        ref = idx.clone()
        idx.fill_(-9)
        graph.replay()
        torch.cuda.synchronize()
        if torch.equal(idx, ref):
            times, launch = timed(graph.replay), "cuda_graph"
    except Exception as exc:  # noqa: BLE001  (reported in the line)
        torch.cuda.synchronize()
        launch = f"direct ({type(exc).__name__}: {exc})"[:200]
    if times is None:
        times = timed(step)
    ms = statistics.median(times)
    return {"ms_per_step": ms, "value": B * L / (ms * 1e-3), "unit": "layer-steps/s",
            "step_launch": launch, "steps": K, "warmup": W,
            "indices_equal_grouped_step": bool(same), "out_rel_l2_vs_grouped_step": err,
            "note": ("context row: every layer's index step and attention after the previous "
                     "layer's (csa2_index_full / csa2_index_reindex / csa2_sparse_attn_decode "
                     "per layer); the headline groups them (one scan + select DAG, one "
                     "attention launch for all layers)")}


def time_context_parallel(csa2, wl, bufs, grp, stream, flush_l2, K, W, world=8):
    """The context-parallel decode step with every sequence cut into `world`
    shards, all run on this one GPU (LocalComm: the shards' kernels back to
    back, each exchange one device copy): its time per step, and whether its
    indices, pool and output equal the one-device step's on the same inputs."""
    import torch
    from fp4_kv_cache_quantize_b200 import cp
    codes, scales, idxk, n_rows, pt, q_idx, w_h, q, swa, swa_len = bufs
    S = cp.shard_rows_for(int(wl.n_rows.max()), world)
    if pt is None and wl.B > 1 and wl.seq_stride < world * S:
        return {"skipped": "contiguous layout narrower than world x shard_rows"}
    ranks = [cp.CPRank(cp.local_view(codes, scales, idxk, rank=r, world=world, shard_rows=S,
                                     batch=wl.B, seq_stride=max(wl.seq_stride, world * S),
                                     page_table=pt),
                       rank=r, world=world, shard_rows=S, n_layers=wl.L, top_k=wl.top_k,
                       pool_blocks=wl.pool_blocks) for r in range(world)]
    comm = cp.LocalComm(world)
    sm = csa2.D ** -0.5

    def step():
        cp.cp_layer_group(ranks, comm, wl.modes, n_rows, q_idx, w_h, q, swa, swa_len,
                          sm_scale=sm)

    for _ in range(W):
        step()
    torch.cuda.synchronize()
    for r in ranks:
        csa2.csa2_sync_status(r.ws)
    same = all(torch.equal(r.idx, grp.idx) and torch.equal(r.idx_count, grp.idx_count)
               for r in ranks)
    if wl.pool_blocks:
        same = same and all(torch.equal(r.pool, grp.pool) for r in ranks)
    a, b = ranks[0].out.double(), grp.out.double()
    err = float((a - b).norm() / max(float(b.norm()), 1e-30))

    def timed(run):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]
        for i in range(K):
            flush_l2()
            ev[i][0].record(stream)
            run()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        return sum(x.elapsed_time(y) for x, y in ev) / K

    ms_direct = timed(step)
    # the same step as one CUDA graph: the shards' launches without Python in between
    ms_graph, graph_note = None, None
    try:
        ref = [r.idx.clone() for r in ranks]
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        torch.cuda.synchronize()
        for r in ranks:
            r.idx.fill_(-9)
        graph.replay()
        torch.cuda.synchronize()
        if all(torch.equal(r.idx, x) for r, x in zip(ranks, ref)):
            ms_graph = timed(graph.replay)
        else:
            graph_note = "graph replay differs from direct launches"
    except Exception as exc:  # noqa: BLE001  (reported in the line)
        torch.cuda.synchronize()
        graph_note = f"{type(exc).__name__}: {exc}"[:200]
    # this library's kernel launches per shard and step (the exchanges' copies excluded)
    modes, hsi = [int(m) for m in wl.modes], wl.pool_blocks > 0
    # (local rows, one filter launch for every layer, attention partial and its
    # local merge, combine; per scan: scan, pool select, block filter, the
    # regroup when batch > 1, and per chunk of at most CP_MAX_JOBS jobs one
    # rescore, one export and one merge launch)
    per_shard = 1 + 1 + 3
    for l, m in enumerate(modes):
        if m == 2 or (m == 1 and hsi):
            continue
        jobs = 1
        if hsi and m == 0:
            for x in modes[l + 1:]:
                if x == 0:
                    break
                jobs += x == 1
        chunks = -(-jobs // csa2.CP_MAX_JOBS)
        per_shard += 3 + (1 if wl.B > 1 and world > 1 else 0) + 3 * chunks
    out = {"world": world, "shard_rows": S, "ms_per_step_one_gpu_emulation": ms_direct,
           "ms_per_step_one_gpu_emulation_graph": ms_graph,
           "launches_per_shard": per_shard, "steps": K, "warmup": W,
           "indices_and_pool_equal_one_device": bool(same),
           "out_rel_l2_vs_one_device": err,
           "note": (f"{world} shards of every sequence run back to back on one GPU, each "
                    "exchange a device copy; the time is the sum over shards plus the "
                    "replicated merges, not a multi-GPU step time; the first figure launches "
                    "from Python, the second replays the step as one CUDA graph")}
    if graph_note:
        out["graph"] = graph_note
    return out


# ------------------------------------------------------------ other configs
QUANT_BYTES_PER_ROW = 1024 + 256 + 32    # bf16 row in, FP4 codes + E4M3 scales out


def sub_workload(wl, S: int):
    """The first S sequences of a workload (same row pool, same seeds)."""
    import dataclasses
    pt = None if wl.page_table is None else np.ascontiguousarray(wl.page_table[:S])
    sub = dataclasses.replace(wl, B=S, n_rows=wl.n_rows[:S].copy(), page_table=pt)
    for name in ("q_idx", "w_h", "q", "swa"):
        setattr(sub, name, np.ascontiguousarray(getattr(wl, name)[:, :S]))
    sub.swa_len = wl.swa_len[:S].copy()
    sub.w_idx = wl.w_idx
    sub.planted = getattr(wl, "planted", None)
    return sub


def oracle_sample_time(wl, idxk_host, S: int):
    """The oracle's layer group on the first S sequences of the workload, on
    one host core: (seconds, S).  Main-KV codes are left zero: the oracle's
    work (full scoring, full sorts, fp64 attention over every selected row)
    does not depend on their values, and regenerating the selected rows of a
    shuffled multi-GB page pool would dominate the sample."""
    import oracle
    sub = sub_workload(wl, S)
    dm = oracle.dims()
    kv = oracle.KV(np.zeros((wl.pool_rows, 256), np.uint8), np.zeros((wl.pool_rows, 32), np.uint8),
                   idxk_host, seq_stride=wl.seq_stride, page_table=sub.page_table)
    t0 = time.perf_counter()
    oracle.layer_group(kv, dm, sub.n_rows, sub.modes, sub.q_idx, sub.w_h, sub.q, sub.swa,
                       sub.swa_len, top_k=sub.top_k, pool_blocks=sub.pool_blocks)
    return time.perf_counter() - t0, S


def setup_device_workload(csa2, wl, dev):
    """Device copies of a workload: its FP4 cache packed by the library's
    pack kernel from the seeded bf16 rows, its indexer K and per-layer
    inputs, a layer group and its workspace."""
    import torch

    def to_dev(a):
        a = np.ascontiguousarray(a)
        t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
        return t.to(dev)

    rows = wl.pool_rows
    codes = torch.empty((rows, 256), dtype=torch.uint8, device=dev)
    scales = torch.empty((rows, 32), dtype=torch.uint8, device=dev)
    idxk = torch.empty((rows, 64), dtype=torch.int16, device=dev)
    for r0, xc, kc in wl.iter_chunks():
        n = len(xc)
        csa2.csa2_quantize_fp4(to_dev(xc).view(torch.bfloat16), codes[r0:r0 + n],
                               scales[r0:r0 + n])
        idxk[r0:r0 + n] = to_dev(kc)
    n_rows = to_dev(wl.n_rows.astype(np.int32))
    pt = None if wl.page_table is None else to_dev(wl.page_table)
    kv = csa2.KVCache(codes, scales, idxk, n_rows, max_rows=int(wl.n_rows.max()),
                      seq_stride=wl.seq_stride, page_table=pt)
    bufs = dict(q_idx=to_dev(wl.q_idx), w_h=to_dev(wl.w_h), q=to_dev(wl.q), swa=to_dev(wl.swa),
                swa_len=to_dev(wl.swa_len))
    grp = csa2.LayerGroup(kv, wl.modes, bufs["q_idx"], bufs["w_h"], bufs["q"], bufs["swa"],
                          bufs["swa_len"], top_k=wl.top_k, pool_blocks=wl.pool_blocks)
    ws = csa2.workspace(grp.workspace_size(), device=dev)
    csa2.csa2_workspace_init(ws)
    return dict(codes=codes, scales=scales, idxk=idxk, n_rows=n_rows, pt=pt, kv=kv, grp=grp,
                ws=ws, **bufs)


def units_of(wl) -> int:
    return int(wl.B * wl.L)


def time_back_to_back(csa2, wl, kv, bufs, ws, stream, K, W, copies: int = 3):
    """Decode steps launched back to back, as a serving loop runs them, with
    no L2 flush: the step's large inputs are kept out of L2 by rotating over
    `copies` copies of the cache (each step streams its copy's indexer K,
    larger than L2, and the copy it reads was last touched `copies` steps
    earlier).  One event pair around all K steps.  Returns ms per step and
    whether every copy's step reproduces the first copy's outputs."""
    import torch
    q_idx, w_h, q, swa, swa_len = bufs
    groups, caches = [], []
    for i in range(copies):
        if i == 0:
            kvi = kv
        else:
            c = (kv.codes.clone(), kv.scales.clone(), kv.idx_k.clone())
            caches.append(c)
            kvi = csa2.KVCache(c[0], c[1], c[2], kv.n_rows, max_rows=int(kv.view.max_rows),
                               seq_stride=int(kv.view.seq_stride), page_table=kv.page_table)
        groups.append(csa2.LayerGroup(kvi, wl.modes, q_idx, w_h, q, swa, swa_len,
                                      top_k=wl.top_k, pool_blocks=wl.pool_blocks))
    wss = [ws] + [csa2.workspace(groups[i].workspace_size(), device=q.device)
                  for i in range(1, copies)]
    for w_ in wss[1:]:
        csa2.csa2_workspace_init(w_)
    runs = []
    for g, w_ in zip(groups, wss):
        csa2.csa2_layer_group(g, w_)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            csa2.csa2_layer_group(g, w_)
        runs.append(graph.replay)
    for i in range(W * copies):
        runs[i % copies]()
    torch.cuda.synchronize()
    same = all(torch.equal(g.idx, groups[0].idx) and torch.equal(g.out, groups[0].out)
               for g in groups[1:])
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(K):
        runs[i % copies]()
    e1.record(stream)
    torch.cuda.synchronize()
    for w_ in wss:
        csa2.csa2_sync_status(w_)
    ms = e0.elapsed_time(e1) / K
    del runs, groups, caches
    return ms, same


def time_workload(csa2, k, dev, stream, flush_l2, K, W, with_cpu, cpu_seqs):
    """A whole layer-group step of config k (the 8 x 131,072 HSI group or the
    64 ragged paged sequences), timed like the headline step: one CUDA graph
    per step, L2 flushed between steps, events around each step; a traced
    pass gives the scan's own duration for its roofline; the oracle runs on
    the first cpu_seqs sequences."""
    import torch
    from fp4_kv_cache_quantize_b200 import synth
    wl = synth.config(k)
    d = setup_device_workload(csa2, wl, dev)
    grp, ws = d["grp"], d["ws"]
    for _ in range(W):
        csa2.csa2_layer_group(grp, ws)
    torch.cuda.synchronize()
    csa2.csa2_sync_status(ws)
    launch = "direct"
    run = lambda: csa2.csa2_layer_group(grp, ws)  # noqa: E731
    try:
        ref = grp.idx.clone()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            csa2.csa2_layer_group(grp, ws)
        torch.cuda.synchronize()
        grp.idx.fill_(-9)
        graph.replay()
        torch.cuda.synchronize()
        if torch.equal(grp.idx, ref):
            run, launch = graph.replay, "cuda_graph"
    except Exception as exc:  # noqa: BLE001  (reported in the line)
        torch.cuda.synchronize()
        launch = f"direct ({type(exc).__name__}: {exc})"[:200]
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    for i in range(K):
        flush_l2()
        ev[i][0].record(stream)
        run()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    csa2.csa2_sync_status(ws)
    times = sorted(a.elapsed_time(b) for a, b in ev)
    ms = sum(times) / K
    try:
        bms, bsame = time_back_to_back(csa2, wl, d["kv"], (d["q_idx"], d["w_h"], d["q"], d["swa"],
                                                          d["swa_len"]), ws, stream, K, W)
        b2b = {"ms_per_step": bms, "value": units_of(wl) / (bms * 1e-3), "copies_agree": bool(bsame)}
    except Exception as exc:  # noqa: BLE001  (reported in the line)
        b2b = {"error": f"{type(exc).__name__}: {exc}"[:300]}
        torch.cuda.synchronize()
    # traced pass: the scan's duration
    n_ev, KT = 32, min(K, 10)
    tev = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev * KT)]
    for e in tev:
        e.record(stream)
    torch.cuda.synchronize()
    scan_ms, stages = [], {}
    for i in range(KT):
        tr = csa2.Trace(tev[i * n_ev:(i + 1) * n_ev])
        flush_l2()
        csa2.csa2_trace_set(tr)
        csa2.csa2_layer_group(grp, ws)
        csa2.csa2_trace_set(None)
        torch.cuda.synchronize()
        names = tr.names()
        for j in range(len(names) - 1):
            dt = tr.events[j].elapsed_time(tr.events[j + 1])
            stages[names[j]] = stages.get(names[j], 0.0) + dt * 1e3 / KT
            if names[j] == "scan":
                scan_ms.append(dt)
    ab = algorithmic_bytes(wl)
    peak, peak_kind = measured_peaks()
    units = wl.B * wl.L
    out = {"workload": wl.name, "value": units / (ms * 1e-3), "unit": UNIT, "ms_per_step": ms,
           "steps": K, "warmup": W, "step_launch": launch,
           "step_ms_p10_p50_p90": [float(np.percentile(times, p)) for p in (10, 50, 90)],
           "algorithmic_bytes_per_step": ab["total"],
           "hbm_gbs_algorithmic": ab["total"] / (ms * 1e-3) / 1e9,
           "frac_of_measured_hbm": ab["total"] / (ms * 1e-3) / 1e9 / peak,
           "stage_us": stages, "back_to_back": b2b, "config": config_dict(wl)}
    if scan_ms:
        t_scan = sum(scan_ms) / len(scan_ms) * 1e-3
        out["roofline"] = {"bound": "hbm", "kernel": "score_scan_kernel",
                           "achieved": ab["scan"] / t_scan / 1e9, "peak": peak,
                           "peak_kind": peak_kind, "unit": "GB/s",
                           "frac": ab["scan"] / t_scan / 1e9 / peak, "traffic": None,
                           "algorithmic_bytes_per_launch": ab["scan"]}
    if with_cpu:
        S = min(cpu_seqs, wl.B)
        idxk_host = d["idxk"].cpu().numpy().view(np.uint16)
        dt, S = oracle_sample_time(wl, idxk_host, S)
        out["cpu_baseline"] = {"value": S * wl.L / dt, "unit": UNIT, "cores": 1,
                               "kind": "oracle",
                               "sample": (f"one step of the first {S} of the {wl.B} sequences "
                                          f"of {wl.name} on one host core (fp64 C oracle; "
                                          "main-KV codes zero, the oracle's work does not "
                                          "depend on them)")}
    del d, grp, ws
    torch.cuda.empty_cache()
    return out


def time_quant(csa2, dev, stream, K, W, with_cpu):
    """The FP4 quantise / dequantise microbenchmark: 1,048,576 x 512 bf16
    rows (0.1% of elements x50) packed to E2M1 codes and E4M3 scales by one
    launch, and unpacked again by one launch.  The 1 GiB input exceeds L2,
    so calls run back to back between two events."""
    import torch
    from fp4_kv_cache_quantize_b200 import synth
    wl = synth.config(1)
    rows = wl.pool_rows
    x = torch.empty((rows, 512), dtype=torch.int16, device=dev)
    for c in range(wl.n_chunks):
        xc = wl.x_chunk(c)
        r0 = c * synth.CHUNK_ROWS
        x[r0:r0 + len(xc)] = torch.from_numpy(xc.view(np.int16)).to(dev)
    xb = x.view(torch.bfloat16)
    codes = torch.empty((rows, 256), dtype=torch.uint8, device=dev)
    scales = torch.empty((rows, 32), dtype=torch.uint8, device=dev)
    y = torch.empty((rows, 512), dtype=torch.bfloat16, device=dev)
    nbytes = rows * QUANT_BYTES_PER_ROW
    peak, peak_kind = measured_peaks()
    out = {"workload": wl.name, "rows": rows, "channels": 512,
           "algorithmic_bytes_per_launch": nbytes}
    for name, fn in (("quantize", lambda: csa2.csa2_quantize_fp4(xb, codes, scales)),
                     ("dequantize", lambda: csa2.csa2_dequantize_fp4(codes, scales, y))):
        for _ in range(W):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(K):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        t = e0.elapsed_time(e1) / K * 1e-3
        gbs = nbytes / t / 1e9
        out[name] = {"us_per_launch": t * 1e6, "value": gbs, "unit": "GB/s",
                     "roofline": {"bound": "hbm", "kernel": f"fp4_{'pack' if name == 'quantize' else 'unpack'}_kernel",
                                  "achieved": gbs, "peak": peak, "peak_kind": peak_kind,
                                  "unit": "GB/s", "frac": gbs / peak,
                                  "traffic": profile_value("fp4_quant_1Mx512.md",
                                                           f"dram_bytes_per_launch_{name}")},
                     "timing": f"{K} back-to-back launches after {W}, CUDA events (1 GiB input > L2)"}
    if with_cpu:
        import oracle
        S = 16384
        xs = wl.x_chunk(0)
        for c in range(1, S // synth.CHUNK_ROWS):
            xs = np.concatenate([xs, wl.x_chunk(c)])
        t0 = time.perf_counter()
        oracle.quantize_fp4(xs)
        dt = time.perf_counter() - t0
        out["cpu_baseline"] = {"value": S * QUANT_BYTES_PER_ROW / dt / 1e9, "unit": "GB/s",
                               "cores": 1, "kind": "oracle",
                               "sample": f"the oracle's quantiser on the first {S} rows"}
    del x, codes, scales, y
    torch.cuda.empty_cache()
    return out


def run_gpu(args, wl, rank, world):
    import torch

    from fp4_kv_cache_quantize_b200 import csa2

    local = int(os.environ.get("LOCAL_RANK", 0))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import torch.distributed as dist_
        import datetime
        dist_.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = dist_

    def barrier():
        if dist:
            dist.barrier()
        torch.cuda.synchronize()

    if args.quant_only:  # the FP4 quantise / dequantise leg alone (its own line)
        stream = torch.cuda.current_stream()
        q = time_quant(csa2, dev, stream, args.steps, args.warmup,
                       rank == 0 and world == 1 and not args.no_cpu)
        if rank == 0:
            print(json.dumps({"metric": "FP4 quantise / dequantise GB/s (algorithmic bytes)",
                              "n_gpus": world, **q}), flush=True)
        return

    def to_dev(a):
        a = np.ascontiguousarray(a)
        t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
        return t.to(dev)

    # ---- setup: FP4 cache via the library's pack kernel, indexer K, inputs
    rows = wl.pool_rows
    codes = torch.empty((rows, 256), dtype=torch.uint8, device=dev)
    scales = torch.empty((rows, 32), dtype=torch.uint8, device=dev)
    idxk = torch.empty((rows, 64), dtype=torch.int16, device=dev)
    for r0, xc, kc in wl.iter_chunks():
        n = len(xc)
        csa2.csa2_quantize_fp4(to_dev(xc).view(torch.bfloat16), codes[r0:r0 + n],
                               scales[r0:r0 + n])
        idxk[r0:r0 + n] = to_dev(kc)
    n_rows = to_dev(wl.n_rows.astype(np.int32))
    pt = None if wl.page_table is None else to_dev(wl.page_table)
    kv = csa2.KVCache(codes, scales, idxk, n_rows, max_rows=int(wl.n_rows.max()),
                      seq_stride=wl.seq_stride, page_table=pt)
    q_idx, w_h, q = to_dev(wl.q_idx), to_dev(wl.w_h), to_dev(wl.q)
    swa, swa_len = to_dev(wl.swa), to_dev(wl.swa_len)
    grp = csa2.LayerGroup(kv, wl.modes, q_idx, w_h, q, swa, swa_len, top_k=wl.top_k,
                          pool_blocks=wl.pool_blocks)
    ws = csa2.workspace(grp.workspace_size(), device=dev)
    csa2.csa2_workspace_init(ws)
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(64 << 20, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream()

    def flush_l2():
        # write 256 MiB (evicts the previous step's lines), then read another
        # 256 MiB so that L2 is left holding clean lines: no write-back of the
        # flush competes with the next step's reads.
        flush_w.zero_()
        flush_r.sum()

    def step():
        csa2.csa2_layer_group(grp, ws)

    for _ in range(args.warmup):
        step()
    csa2.csa2_sync_status(ws)

    def capture(g_grp):
        """One decode step as a CUDA graph (its launches keep their
        programmatic-serialisation edges), or the exception that stopped it."""
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                csa2.csa2_layer_group(g_grp, ws)
            torch.cuda.synchronize()
            return graph
        except Exception as exc:  # noqa: BLE001  (reported, then direct launches)
            torch.cuda.synchronize()
            return exc

    ref_idx, ref_out = grp.idx.clone(), grp.out.clone()
    graph = capture(grp)
    if isinstance(graph, torch.cuda.CUDAGraph):
        grp.idx.fill_(-9)
        graph.replay()
        torch.cuda.synchronize()
        csa2.csa2_sync_status(ws)
        assert torch.equal(grp.idx, ref_idx) and torch.equal(grp.out, ref_out), \
            "graph replay differs from direct launches"
        step_launch = "cuda_graph"
        run_step = graph.replay
    else:
        step_launch = f"direct ({type(graph).__name__}: {graph})"[:200]
        run_step = step

    # ---- timed device loop
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    sampler = ClockSampler(local)
    barrier()
    with sampler:
        for i in range(K):
            flush_l2()
            ev[i][0].record(stream)
            run_step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    barrier()
    csa2.csa2_sync_status(ws)
    times = [a.elapsed_time(b) for a, b in ev]   # ms
    t_step = max_over_ranks(sum(times) / K, dist, dev)

    # ---- the same steps back to back (no flush; the cache rotates over three
    # copies so that every step's large inputs are cold in L2)
    try:
        b2b_ms, b2b_same = time_back_to_back(csa2, wl, kv, (q_idx, w_h, q, swa, swa_len), ws,
                                             stream, K, args.warmup)
        b2b_ms = max_over_ranks(b2b_ms, dist, dev)
        b2b = {"ms_per_step": b2b_ms, "value": job_throughput(wl.B * wl.L, world, b2b_ms),
               "unit": UNIT, "copies_agree": bool(b2b_same),
               "timing": (f"{K} steps back to back between two events after warm-up, no L2 "
                          "flush: the steps rotate over three copies of the cache, so every "
                          "step streams indexer K that the two steps before it did not touch "
                          "(3 x 134 MB > the 126 MB L2)")}
    except Exception as exc:  # noqa: BLE001  (reported in the line)
        b2b = {"error": f"{type(exc).__name__}: {exc}"[:300]}
        torch.cuda.synchronize()

    # ---- traced pass: per-launch events for the stage breakdown and roofline
    n_ev = 32
    tev = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev * K)]
    for e in tev:
        e.record(stream)
    torch.cuda.synchronize()
    traces = []
    for i in range(K):
        tr = csa2.Trace(tev[i * n_ev:(i + 1) * n_ev])
        flush_l2()
        csa2.csa2_trace_set(tr)
        step()
        csa2.csa2_trace_set(None)
        traces.append(tr)
    torch.cuda.synchronize()
    stage_tot, stage_n, launches = {}, {}, 0
    for tr in traces:
        names = tr.names()
        launches = len(names) - 1
        for j in range(len(names) - 1):
            d = tr.events[j].elapsed_time(tr.events[j + 1])
            stage_tot[names[j]] = stage_tot.get(names[j], 0.0) + d
            stage_n[names[j]] = stage_n.get(names[j], 0) + 1
    stage_us_step = {k: 1e3 * v / K for k, v in stage_tot.items()}       # per step
    stage_us_launch = {k: 1e3 * v / stage_n[k] for k, v in stage_tot.items()}  # per launch

    # ---- end to end through the C ABI with host buffers
    h_q_idx = torch.from_numpy(np.ascontiguousarray(wl.q_idx).view(np.int16)).pin_memory()
    h_w = torch.from_numpy(np.ascontiguousarray(wl.w_h)).pin_memory()
    h_q = torch.from_numpy(np.ascontiguousarray(wl.q).view(np.int16)).pin_memory()
    h_out = torch.empty(grp.out.shape, dtype=torch.bfloat16).pin_memory()
    h_idx = torch.empty(grp.idx.shape, dtype=torch.int32).pin_memory()
    h2d = h_q_idx.numel() * 2 + h_w.numel() * 4 + h_q.numel() * 2
    d2h = h_out.numel() * 2 + h_idx.numel() * 4
    # Steps run back to back with the copies overlapped: the host->device
    # copy of step i+1's inputs and the device->host copy of step i-1's
    # results run on their own streams while step i computes (two sets of
    # device input and output buffers).  E2E_UNROLL consecutive steps (their
    # copies and their csa2_layer_group calls, on three streams with the
    # dependencies above) are captured as one CUDA graph, so the host issues
    # one launch per E2E_UNROLL steps and its own speed does not set the
    # step time.  No L2 flush here: every step streams 134 MB of indexer K,
    # more than the 126 MB L2.
    sets = [(q_idx, w_h, q, grp)]
    q_idx2, w_h2, q2 = torch.empty_like(q_idx), torch.empty_like(w_h), torch.empty_like(q)
    grp2 = csa2.LayerGroup(kv, wl.modes, q_idx2, w_h2, q2, swa, swa_len, top_k=wl.top_k,
                           pool_blocks=wl.pool_blocks)
    sets.append((q_idx2, w_h2, q2, grp2))
    csa2.csa2_layer_group(grp2, ws)   # set up outside the capture
    torch.cuda.synchronize()
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    h_outs = [h_out, torch.empty_like(h_out).pin_memory()]
    h_idxs = [h_idx, torch.empty_like(h_idx).pin_memory()]

    def e2e_steps(n):
        """n steps with overlapped copies, issued on the current stream."""
        main = torch.cuda.current_stream()
        fork = torch.cuda.Event()
        fork.record(main)
        ev_done = [fork, fork]
        ev_out = [fork, fork]
        for i in range(n):
            j = i % 2
            d_qi, d_w, d_q, g = sets[j]
            ev_in = torch.cuda.Event()
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_done[j])          # step i-2 no longer reads set j
                d_qi.copy_(h_q_idx, non_blocking=True)
                d_w.copy_(h_w, non_blocking=True)
                d_q.copy_(h_q, non_blocking=True)
                ev_in.record(s_in)
            main.wait_event(ev_in)
            main.wait_event(ev_out[j])               # step i-2's results have left set j
            csa2.csa2_layer_group(g, ws)
            ev_done[j] = torch.cuda.Event()
            ev_done[j].record(main)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[j])
                h_outs[j].copy_(g.out, non_blocking=True)
                h_idxs[j].copy_(g.idx, non_blocking=True)
                ev_out[j] = torch.cuda.Event()
                ev_out[j].record(s_out)
        main.wait_event(ev_out[0])
        main.wait_event(ev_out[1])

    E2E_UNROLL = 10
    reps = max(1, K // E2E_UNROLL)
    e2e_graph = None
    if step_launch == "cuda_graph":
        try:
            e2e_graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(e2e_graph):
                e2e_steps(E2E_UNROLL)
            torch.cuda.synchronize()
        except Exception:  # noqa: BLE001  (direct launches below)
            torch.cuda.synchronize()
            e2e_graph = None
    e2e_launch = f"cuda_graph of {E2E_UNROLL} steps" if e2e_graph else "direct"
    for _ in range(2):  # warm-up
        e2e_graph.replay() if e2e_graph else e2e_steps(E2E_UNROLL)
    t0e, t1e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier()
    t0e.record(stream)
    for _ in range(reps):
        e2e_graph.replay() if e2e_graph else e2e_steps(E2E_UNROLL)
    t1e.record(stream)
    torch.cuda.synchronize()
    barrier()
    csa2.csa2_sync_status(ws)
    K_e2e = reps * E2E_UNROLL
    t_e2e = max_over_ranks(t0e.elapsed_time(t1e) / K_e2e, dist, dev)
    assert torch.equal(h_idxs[0], grp.idx.cpu()) and torch.equal(h_idxs[1], grp.idx.cpu())

    with_cpu = rank == 0 and world == 1 and not args.no_cpu
    append = time_cache_append(csa2, wl, dev, stream, K, args.warmup, with_cpu)
    multi = time_multi_query(csa2, wl, kv, dev, stream, flush_l2, max(10, K // 4), args.warmup,
                             with_cpu)
    prefill = time_multi_query(csa2, wl, kv, dev, stream, flush_l2, 5, 3, with_cpu, Q=64)
    prefill["note"] = ("chunked prefill of 64 new tokens; the scan runs 8 passes of 8 queries "
                       "(MMA N = 64)")
    def quiet_sync():
        # a failed optional measurement must not take the headline line with it
        try:
            torch.cuda.synchronize()
        except Exception:  # noqa: BLE001
            pass

    try:
        seq = time_layer_sequential(csa2, wl, kv, (q_idx, w_h, q, swa, swa_len), grp, stream,
                                    flush_l2, 20, 3)
    except Exception as exc:  # noqa: BLE001  (reported in the line)
        seq = {"error": f"{type(exc).__name__}: {exc}"[:300]}
        quiet_sync()
    try:
        cpar = time_context_parallel(
            csa2, wl, (codes, scales, idxk, n_rows, pt, q_idx, w_h, q, swa, swa_len), grp, stream,
            flush_l2, 10, 3)
    except Exception as exc:  # noqa: BLE001  (reported in the line)
        cpar = {"error": f"{type(exc).__name__}: {exc}"[:300]}
        quiet_sync()

    others = {}
    for key_, fn in (("fp4_quant_1Mx512", lambda: time_quant(csa2, dev, stream, 20, 3, with_cpu)),
                     ("hsi_group_b8_128k", lambda: time_workload(csa2, 2, dev, stream, flush_l2,
                                                                 max(10, K // 2), 3, with_cpu, 8)),
                     ("ragged_paged_64seq_r2", lambda: time_workload(
                         csa2, 4, dev, stream, flush_l2, max(10, K // 2), 3, with_cpu, 4))):
        if args.skip_configs:
            break
        try:
            others[key_] = fn()
        except Exception as exc:  # noqa: BLE001  (reported in the line)
            others[key_] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
            quiet_sync()

    units = wl.B * wl.L
    value = job_throughput(units, world, t_step)
    ab = algorithmic_bytes(wl)
    peak, peak_kind = measured_peaks()
    scan_us = stage_us_launch.get("scan")
    roof = None
    if scan_us:
        achieved = ab["scan"] / max(1, int((wl.modes == 0).sum())) / (scan_us * 1e-6) / 1e9
        roof = {"bound": "hbm", "kernel": "score_scan_kernel", "achieved": achieved,
                "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                "frac": achieved / peak, "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                "traffic": scan_traffic_from_profile(),
                "algorithmic_bytes_per_launch": ab["scan"] // max(1, int((wl.modes == 0).sum()))}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        dt = oracle_step_time(wl)
        cpu = {"value": units / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"one full decode step of {wl.name} on one host core (fp64 C oracle)"}
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": t_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_dict(wl),
            "hbm_gbs_algorithmic": ab["total"] / (t_step * 1e-3) / 1e9,
            "algorithmic_bytes_per_step": ab["total"],
            "step_launch": step_launch,
            "stage_us": stage_us_step,
            "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": job_throughput(units, world, t_e2e), "unit": UNIT,
                    "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                    "ms_per_step": t_e2e,
                    "launch": e2e_launch,
                    "timing": (f"{K_e2e} back-to-back steps through the C ABI; each step's inputs "
                               "copied from pinned host memory and its outputs (attention "
                               "output, indices) copied back, on separate streams overlapping "
                               "the neighbouring steps' compute; every "
                               f"{E2E_UNROLL} steps' copies and calls replayed as one CUDA "
                               "graph; no L2 flush (134 MB of indexer K per step exceeds the "
                               "126 MB L2)")},
            "back_to_back": b2b,
            "configs": others,
            "layer_sequential": seq,
            "next_rows": {"cache_append": append, "multi_query": multi,
                          "prefill_chunk": prefill, "context_parallel": cpar},
            "gpu_launches": int(launches * K),
            "gpu_launches_per_step": int(launches),
            "clocks": sampler.summary(),
            "step_ms_p10_p50_p90": [float(np.percentile(times, p)) for p in (10, 50, 90)]}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="csa2", choices=["csa2", "reference"])
    ap.add_argument("--config", type=int, default=3)
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--skip-configs", action="store_true",
                    help="time only the headline workload (not configs 1, 2 and 4)")
    ap.add_argument("--quant-only", action="store_true",
                    help="time only the FP4 quantise / dequantise leg (1M x 512 rows)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    from fp4_kv_cache_quantize_b200 import synth
    wl = synth.config(args.config)
    if args.impl == "reference":
        run_reference(args, wl, rank)
        return
    run_gpu(args, wl, rank, world)


if __name__ == "__main__":
    main()
