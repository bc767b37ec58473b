"""Host-side logic of bench.py, on the CPU: the algorithmic bytes per step
against the closed forms of the measurement contract (config 0: 4,096
positions, one Full layer and three Reuse layers; config 2: 8 x 131,072, one
Full and one Reindex layer over a 2,048-block pool, 40 layer-steps; config 3:
1M positions, 20 layers), the whole-job throughput, the roofline fraction's
inputs, and the layer-sequential context row's calls (with stand-ins of the
entry points: one index step per Full / Reindex layer, one attention per layer,
every count array on a 16-byte boundary, indices compared with the grouped
step's)."""
import os
import sys
import types

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from fp4_kv_cache_quantize_b200 import synth  # noqa: E402

ATTN = 512 * 288 + 128 * 512 + 2 * 16384 + 2048


def test_attention_bytes_per_layer_and_sequence():
    assert bench.ATTN_BYTES == ATTN == 247808


def test_algorithmic_bytes_of_the_workloads():
    assert bench.algorithmic_bytes(synth.config(0))["total"] == 524288 + 4 * ATTN == 1515520
    ab2 = bench.algorithmic_bytes(synth.config(2))
    assert ab2["scan"] == 8 * 131072 * 128
    assert ab2["reindex"] == 8 * 16384 * 128
    assert ab2["total"] == 134217728 + 16777216 + 40 * ATTN == 160907264
    ab3 = bench.algorithmic_bytes(synth.config(3))
    assert ab3["scan"] == 134217728 and ab3["reindex"] == 4 * 2097152
    assert ab3["total"] == 147562496


def test_job_throughput_counts_every_rank():
    assert np.isclose(bench.job_throughput(20, 1, 0.0724), 20 / 0.0724e-3, rtol=1e-12)
    assert np.isclose(bench.job_throughput(20, 8, 0.0724), 8 * 20 / 0.0724e-3, rtol=1e-12)


class _Ev:
    def __init__(self, **_):
        pass

    def record(self, *_):
        pass

    def elapsed_time(self, _):
        return 0.25


def _fake_lib(calls):
    def chk(t, shape):
        assert t.is_contiguous() and tuple(t.shape) == tuple(shape), (t.shape, shape)
        assert t.data_ptr() % 16 == 0

    lib = types.SimpleNamespace(D=512)
    lib.workspace = lambda n, device=None: torch.zeros(max(n, 256), dtype=torch.uint8)
    lib.csa2_index_workspace_size = lambda kv, k, p: 256
    lib.csa2_attn_workspace_size = lambda b, n: 256
    lib.csa2_sync_status = lambda ws: None

    def full(kv, qi, w, K, P, idx, cnt, pool, pcnt, ws):
        chk(qi, (kv.batch, 8, 64)), chk(w, (kv.batch, 8)), chk(idx, (kv.batch, K))
        chk(cnt, (kv.batch,)), chk(pool, (kv.batch, P)), chk(pcnt, (kv.batch,))
        idx.copy_(torch.arange(K).repeat(kv.batch, 1))
        cnt.fill_(K)
        calls.append("full")

    def reindex(kv, qi, w, pool, pcnt, stride, K, idx, cnt, ws):
        chk(idx, (kv.batch, K)), chk(cnt, (kv.batch,))
        assert stride == pool.shape[1]
        idx.copy_(torch.arange(K).repeat(kv.batch, 1) + 1)
        cnt.fill_(K - 1)
        calls.append("reindex")

    def attn(q, kv, idx, cnt, K, swa, swa_len, sm, out, ws):
        chk(q, (kv.batch, 16, 512)), chk(idx, (kv.batch, K)), chk(cnt, (kv.batch,))
        chk(swa, (kv.batch, 128, 512)), chk(out, (kv.batch, 16, 512))
        out.fill_(float(idx[0, 0]))
        calls.append("attn")

    lib.csa2_index_full, lib.csa2_index_reindex, lib.csa2_sparse_attn_decode = full, reindex, attn
    return lib


def test_layer_sequential_row_issues_one_step_per_layer(monkeypatch):
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(torch.cuda, "Event", _Ev)

    class NoGraph:
        def __init__(self):
            raise RuntimeError("no graphs on the CPU")

    monkeypatch.setattr(torch.cuda, "CUDAGraph", NoGraph)
    for B in (1, 3):
        wl = synth.make("seq", seed=1, B=B, n_rows=[1000] * B, modes=synth.DECODER_20)
        L, K = wl.L, wl.top_k
        bufs = (torch.zeros((L, B, 8, 64), dtype=torch.int16), torch.zeros((L, B, 8)),
                torch.zeros((L, B, 16, 512), dtype=torch.bfloat16),
                torch.zeros((L, B, 128, 512), dtype=torch.uint8), torch.zeros(B, dtype=torch.int32))
        grp = types.SimpleNamespace(idx=torch.zeros((L, B, K), dtype=torch.int32),
                                    idx_count=torch.zeros((L, B), dtype=torch.int32),
                                    out=torch.zeros((L, B, 16, 512), dtype=torch.bfloat16))
        src = 0
        for l, m in enumerate(wl.modes):
            if m != 2:
                src = l
                grp.idx[l] = torch.arange(K) + (1 if m == 1 else 0)
                grp.idx_count[l] = K - (1 if m == 1 else 0)
            else:
                grp.idx[l], grp.idx_count[l] = grp.idx[src], grp.idx_count[src]
            grp.out[l] = float(grp.idx[l][0, 0])
        calls = []
        r = bench.time_layer_sequential(_fake_lib(calls), wl, types.SimpleNamespace(batch=B), bufs,
                                        grp, None, lambda: None, 4, 3)
        steps = 3 + 4
        assert calls.count("full") == steps * int((wl.modes == 0).sum())
        assert calls.count("reindex") == steps * int((wl.modes == 1).sum())
        assert calls.count("attn") == steps * L
        assert r["indices_equal_grouped_step"] and r["out_rel_l2_vs_grouped_step"] == 0.0
        assert r["step_launch"].startswith("direct") and r["ms_per_step"] == 0.25
        assert np.isclose(r["value"], B * L / 0.25e-3)


def test_reference_arm_counts_fit_the_budget():
    """The reference arm runs the requested warm-up and timed steps when they
    fit its budget, and as many as fit otherwise (at least one of each)."""
    import bench
    assert bench.reference_counts(3, 20, 0.5, budget_s=150) == (3, 20)
    w, k = bench.reference_counts(10, 200, 3.8, budget_s=150)
    assert (w, k) == (3, 36) and (w + k) * 3.8 <= 150 + 3.8
    assert bench.reference_counts(3, 20, 400.0, budget_s=150) == (1, 1)
    assert bench.reference_counts(0, 0, 1.0, budget_s=150) == (1, 1)
