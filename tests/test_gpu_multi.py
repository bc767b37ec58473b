"""GPU parity of the multi-query (draft verification) decode step: one
csa2_layer_group call with n_query = Q against the oracle's multi-query step.
Every (sequence, query) pair is checked like a single decode step with its
own visibility: indices of every layer (ties within 1e-5 of the k-th score),
the HSI pool (ties within 1e-5 of the pool threshold) and the attention
output (relative L2 <= 5e-3)."""
import numpy as np
import pytest
import torch

from fp4_kv_cache_quantize_b200 import synth
from gpu_helpers import ATTN_RTOL, DeviceWorkload, bf16_to_f64, check_selection, dev, rel_l2

pytestmark = pytest.mark.gpu
FULL, REINDEX, REUSE = 0, 1, 2


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp4_kv_cache_quantize_b200 import csa2
    return csa2


def mq_inputs(Q, L, B, swa_len, seed):
    rng = np.random.default_rng(seed)
    bf = lambda a: synth.to_bf16_bits(np.asarray(a, np.float32))  # noqa: E731
    return dict(q_idx=bf(rng.standard_normal((L, B, Q, 8, 64))),
                w=rng.uniform(0, 1, (L, B, Q, 8)).astype(np.float32),
                q=bf(rng.standard_normal((L, B, Q, 16, 512))),
                swa=synth.to_e4m3_bits(rng.standard_normal((L, B, 128 + Q - 1, 512)).astype(
                    np.float32)),
                swa_len=np.asarray(swa_len, np.int32))


def run_and_check(lib, orc, n_rows, Q, modes, swa_len, pool_blocks, seed, paged=False):
    L, B = len(modes), len(n_rows)
    wl = synth.make("mq", seed=seed, B=B, n_rows=n_rows, modes=modes, pool_blocks=pool_blocks,
                    paged=paged)
    dw = DeviceWorkload(lib, wl, orc)
    m = mq_inputs(Q, L, B, swa_len, seed + 1)
    VB = B * Q
    grp = lib.LayerGroup(dw.kv, modes, dev(m["q_idx"].reshape(L, VB, 8, 64)),
                         dev(m["w"].reshape(L, VB, 8)), dev(m["q"].reshape(L, VB, 16, 512)),
                         dev(m["swa"]), dev(m["swa_len"]), top_k=512, pool_blocks=pool_blocks,
                         n_query=Q)
    ws = lib.workspace(grp.workspace_size())
    lib.csa2_layer_group(grp, ws)
    lib.csa2_sync_status(ws)
    kv = dw.oracle_kv(orc)
    dm = orc.dims()
    ref = orc.layer_group_multi(kv, dm, wl.n_rows, Q, modes, m["q_idx"], m["w"], m["q"],
                                m["swa"], m["swa_len"], top_k=512, pool_blocks=pool_blocks,
                                sm_scale=float(np.float32(512 ** -0.5)))
    idx = grp.idx.cpu().numpy().reshape(L, B, Q, 512)
    cnt = grp.idx_count.cpu().numpy().reshape(L, B, Q)
    out = bf16_to_f64(grp.out).reshape(L, B, Q, 16, 512)
    gpool = grp.pool.cpu().numpy().reshape(B, Q, -1)
    gpc = grp.pool_count.cpu().numpy().reshape(B, Q)
    for b in range(B):
        for t in range(Q):
            C = max(0, int(wl.n_rows[b]) - (Q - 1 - t))
            pool_ok = None
            for l in range(L):
                if modes[l] in (FULL, REINDEX):
                    s_l = orc.scores(kv, dm, b, C, m["q_idx"][l, b, t], m["w"][l, b, t])
                if modes[l] == FULL:
                    cand = np.arange(C)
                    if pool_blocks:
                        bm = orc.block_max(s_l, 8)
                        check_selection(gpool[b, t], int(gpc[b, t]),
                                        ref["pool"][b, t, :ref["pool_count"][b, t]],
                                        lambda j: bm[j], pool_blocks,
                                        cand_positions=np.arange(len(bm)), what=f"pool {b},{t}")
                        thr = np.sort(bm)[::-1][min(pool_blocks, len(bm)) - 1] if len(bm) else 0
                        pool_ok = lambda pos, bm=bm, thr=thr: np.abs(bm[pos // 8] - thr) <= 1e-5 * abs(thr)  # noqa: E731,E501
                elif modes[l] == REINDEX:
                    if pool_blocks:
                        op = ref["pool"][b, t, :ref["pool_count"][b, t]]
                        cand = np.array([p for j in op for p in range(8 * j, min(8 * j + 8, C))],
                                        dtype=np.int64)
                    else:
                        cand = np.arange(C)
                want = ref["idx"][l, b, t, :ref["idx_count"][l, b, t]]
                check_selection(idx[l, b, t], int(cnt[l, b, t]), want, lambda p: s_l[p], 512,
                                cand_positions=cand,
                                extra_ok=pool_ok if modes[l] == REINDEX else None,
                                what=f"layer {l} ({b},{t})")
                err = rel_l2(out[l, b, t], ref["out"][l, b, t])
                assert err <= ATTN_RTOL, (l, b, t, err)


@pytest.mark.parametrize("Q,n_rows,swa_len", [
    (2, [20000, 9001], [129, 40]),
    (3, [12000, 700], [130, 3]),
    (4, [15000, 3000], [131, 77]),  # the draft count the benchmark's multi-query line times
    (8, [9000, 2050], [135, 100]),
    (20, [3000, 10], [147, 5]),     # three scan passes; early queries of b=1 see nothing
    (64, [2500], [191]),            # chunked prefill: eight scan passes
])
def test_multi_query_group_parity(lib, orc, Q, n_rows, swa_len):
    run_and_check(lib, orc, n_rows, Q, [FULL, REINDEX, REUSE], swa_len, 2048, seed=300 + Q)


def test_multi_query_paged_without_pool(lib, orc):
    run_and_check(lib, orc, [5000, 1300], 4, [FULL, REUSE], [131, 0], 0, seed=410, paged=True)


def test_multi_query_rejects_too_many_queries(lib, orc):
    wl = synth.make("mq", seed=5, B=1, n_rows=[100], modes=[FULL])
    dw = DeviceWorkload(lib, wl, orc)
    Q = 1025
    m = mq_inputs(Q, 1, 1, [10], 6)
    grp = lib.LayerGroup(dw.kv, [FULL], dev(m["q_idx"].reshape(1, Q, 8, 64)),
                         dev(m["w"].reshape(1, Q, 8)), dev(m["q"].reshape(1, Q, 16, 512)),
                         dev(m["swa"]), dev(m["swa_len"]), n_query=Q)
    with pytest.raises(lib.Csa2Error) as e:
        lib.csa2_layer_group(grp, lib.workspace(1 << 20))
    assert e.value.status == 2
