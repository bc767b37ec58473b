"""GPU parity of the indexer (Full scan + HSI pool + Top-k; Reindex) and of
the attention kernel, each through the C ABI, against the CPU oracle."""
import numpy as np
import pytest
import torch

from fp4_kv_cache_quantize_b200 import synth
from gpu_helpers import (ATTN_RTOL, DeviceWorkload, bf16_to_f64, check_selection, dev, rel_l2)

pytestmark = pytest.mark.gpu
FULL, REINDEX, REUSE = 0, 1, 2


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp4_kv_cache_quantize_b200 import csa2
    return csa2


def run_full(lib, dw, layer, top_k, pool_blocks):
    B = dw.wl.B
    idx = torch.full((B, top_k), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    pb = max(pool_blocks, 1)
    pool = torch.full((B, pb), -7, dtype=torch.int32, device="cuda")
    pcnt = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    ws = lib.workspace(lib.csa2_index_workspace_size(dw.kv, top_k, pool_blocks))
    lib.csa2_index_full(dw.kv, dw.q_idx[layer], dw.w[layer], top_k, pool_blocks, idx, cnt,
                        pool if pool_blocks else None, pcnt if pool_blocks else None, ws)
    lib.csa2_sync_status(ws)
    return idx.cpu().numpy(), cnt.cpu().numpy(), pool.cpu().numpy(), pcnt.cpu().numpy()


def check_full(orc, dw, layer, top_k, pool_blocks, idx, cnt, pool, pcnt):
    wl = dw.wl
    kv = dw.oracle_kv(orc)
    dm = orc.dims()
    for b in range(wl.B):
        C = int(wl.n_rows[b])
        s = orc.scores(kv, dm, b, C, wl.q_idx[layer, b], wl.w_h[layer, b])
        want = orc.select_topk(s, top_k)
        check_selection(idx[b], int(cnt[b]), want, lambda p: s[p], top_k,
                        cand_positions=np.arange(C), what=f"full b={b}")
        if pool_blocks:
            bm = orc.block_max(s, 8)
            wp = orc.pool(bm, pool_blocks)
            check_selection(pool[b], int(pcnt[b]), wp, lambda j: bm[j], pool_blocks,
                            cand_positions=np.arange(len(bm)), what=f"pool b={b}")


@pytest.mark.parametrize("n_rows,pool_blocks,paged", [
    ([3000, 777], 2048, False),       # pool larger than the block count
    ([20000, 16391], 2048, False),    # real pool selection, ragged tails
    ([20000, 9], 0, False),           # no HSI pool (encoder style)
    ([5000, 4097, 1], 2048, True),    # paged, C = 1
    ([0, 300, 513], 2048, False),     # empty sequence, C < top_k
])
def test_index_full_parity(lib, orc, n_rows, pool_blocks, paged):
    wl = synth.make("idx", seed=101 + sum(n_rows), B=len(n_rows), n_rows=n_rows,
                    modes=[FULL, REINDEX], pool_blocks=pool_blocks, paged=paged)
    dw = DeviceWorkload(lib, wl, orc)
    out = run_full(lib, dw, 0, 512, pool_blocks)
    check_full(orc, dw, 0, 512, pool_blocks, *out)


@pytest.mark.parametrize("pool_blocks", [2048, 0])
def test_index_full_exact_ties(lib, orc, pool_blocks):
    """Indexer K rows repeat with period 37, so scores and block maxima tie
    exactly (on both sides); the selection must follow the tie rule exactly:
    lower position, lower block id."""
    n_rows = [20000, 3000]
    wl = synth.make("ties", seed=31, B=2, n_rows=n_rows, modes=[FULL], pool_blocks=pool_blocks)
    dw = DeviceWorkload(lib, wl, orc)
    k = dw.idxk_np.copy()
    for b in range(wl.B):
        base = b * wl.seq_stride
        k[base:base + wl.seq_stride] = k[base + np.arange(wl.seq_stride) % 37]
    dw.idxk_np = k
    dw.idxk.copy_(dev(k))
    idx, cnt, pool, pcnt = run_full(lib, dw, 0, 512, pool_blocks)
    kv = dw.oracle_kv(orc)
    for b in range(wl.B):
        s = orc.scores(kv, orc.dims(), b, n_rows[b], wl.q_idx[0, b], wl.w_h[0, b])
        assert np.array_equal(idx[b, :cnt[b]], orc.select_topk(s, 512)), b
        if pool_blocks:
            assert np.array_equal(pool[b, :pcnt[b]], orc.pool(orc.block_max(s, 8), pool_blocks))


@pytest.mark.parametrize("pool_blocks,n_rows", [(2048, [40000, 700]), (0, [40000, 700]),
                                               (2048, [100000, 65])])
def test_index_full_all_scores_equal(lib, orc, pool_blocks, n_rows):
    """A zero indexer query makes every score 0: the whole range ties, so the
    first positions and the first blocks are selected.  At 100,000 rows the
    tied block maxima outnumber what the bounded gather holds, so the block
    selection takes its radix path."""
    wl = synth.make("zero", seed=32, B=2, n_rows=n_rows, modes=[FULL], pool_blocks=pool_blocks)
    dw = DeviceWorkload(lib, wl, orc)
    dw.q_idx.zero_()
    idx, cnt, pool, pcnt = run_full(lib, dw, 0, 512, pool_blocks)
    for b in range(wl.B):
        assert np.array_equal(idx[b, :cnt[b]], np.arange(min(512, n_rows[b]))), b
        if pool_blocks:
            nb = (n_rows[b] + 7) // 8
            assert np.array_equal(pool[b, :pcnt[b]], np.arange(min(pool_blocks, nb))), b


def test_index_full_small_topk_and_pool(lib, orc):
    wl = synth.make("idx", seed=7, B=2, n_rows=[1234, 4321], modes=[FULL], pool_blocks=40)
    dw = DeviceWorkload(lib, wl, orc)
    check_full(orc, dw, 0, 37, 40, *run_full(lib, dw, 0, 37, 40))


@pytest.mark.parametrize("with_pool", [True, False])
def test_index_reindex_parity(lib, orc, with_pool):
    wl = synth.make("rx", seed=55, B=2, n_rows=[30000, 7001], modes=[FULL, REINDEX],
                    pool_blocks=2048 if with_pool else 0)
    dw = DeviceWorkload(lib, wl, orc)
    kv = dw.oracle_kv(orc)
    dm = orc.dims()
    B = wl.B
    # the pool the Reindex layer searches comes from the oracle (an input)
    pools = np.full((B, 2048), -1, np.int32)
    pcnt = np.zeros(B, np.int32)
    for b in range(B):
        s0 = orc.scores(kv, dm, b, int(wl.n_rows[b]), wl.q_idx[0, b], wl.w_h[0, b])
        p = orc.pool(orc.block_max(s0, 8), 2048)
        pools[b, :len(p)] = p
        pcnt[b] = len(p)
    idx = torch.full((B, 512), -7, dtype=torch.int32, device="cuda")
    cnt = torch.zeros((B,), dtype=torch.int32, device="cuda")
    ws = lib.workspace(lib.csa2_index_workspace_size(dw.kv, 512, 0))
    lib.csa2_index_reindex(dw.kv, dw.q_idx[1], dw.w[1], dev(pools) if with_pool else None,
                           dev(pcnt) if with_pool else None, 2048, 512, idx, cnt, ws)
    lib.csa2_sync_status(ws)
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    for b in range(B):
        C = int(wl.n_rows[b])
        s1 = orc.scores(kv, dm, b, C, wl.q_idx[1, b], wl.w_h[1, b])
        if with_pool:
            cand = np.array([p for j in pools[b, :pcnt[b]] for p in range(8 * j, min(8 * j + 8, C))])
        else:
            cand = np.arange(C)
        want = orc.select_topk(s1[cand], 512, cand)
        check_selection(idx[b], int(cnt[b]), want, lambda p: s1[p], 512, cand_positions=cand,
                        what=f"reindex b={b}")
        if with_pool:
            assert set((idx[b, :cnt[b]] // 8).tolist()) <= set(pools[b, :pcnt[b]].tolist())


# ------------------------------------------------------------ attention
@pytest.mark.parametrize("n_rows,swa_len,paged", [
    ([4096, 1000], [128, 128], False),
    ([700, 333, 5000], [128, 77, 0], False),
    ([3000, 64, 0], [128, 1, 128], True),
])
def test_attention_parity(lib, orc, n_rows, swa_len, paged):
    B = len(n_rows)
    wl = synth.make("at", seed=9 + B, B=B, n_rows=n_rows, modes=[FULL], paged=paged,
                    swa_len=swa_len)
    dw = DeviceWorkload(lib, wl, orc)
    kv = dw.oracle_kv(orc)
    dm = orc.dims()
    g = np.random.default_rng(3)
    idx = np.full((B, 512), -1, np.int32)
    cnt = np.zeros(B, np.int32)
    for b in range(B):
        C = int(wl.n_rows[b])
        k = min(512, C) if b != 1 else min(200, C)   # also a partial index set
        sel = np.sort(g.choice(C, k, replace=False)) if k else np.zeros(0, np.int64)
        idx[b, :k] = sel
        cnt[b] = k
    out = torch.zeros((B, 16, 512), dtype=torch.bfloat16, device="cuda")
    ws = lib.workspace(lib.csa2_attn_workspace_size(B, 1))
    scale = 512 ** -0.5
    lib.csa2_sparse_attn_decode(dw.q[0], dw.kv, dev(idx), dev(cnt), 512, dw.swa[0], dw.swa_len,
                                scale, out, ws)
    lib.csa2_sync_status(ws)
    got = bf16_to_f64(out)
    for b in range(B):
        want = orc.attention(kv, dm, b, wl.q[0, b], idx[b, :cnt[b]], wl.swa[0, b],
                             int(wl.swa_len[b]), float(np.float32(scale)))
        if cnt[b] == 0 and wl.swa_len[b] == 0:
            assert np.all(got[b] == 0)
        else:
            assert rel_l2(got[b], want) <= ATTN_RTOL, (b, rel_l2(got[b], want))


def test_attention_device_check_on_bad_index(lib, orc):
    """An index outside the visible range is never dereferenced: the row is
    skipped and csa2_sync_status reports CSA2_ERR_DEVICE_CHECK."""
    wl = synth.make("at", seed=4, B=1, n_rows=[100], modes=[FULL])
    dw = DeviceWorkload(lib, wl, orc)
    idx = np.full((1, 512), -1, np.int32)
    idx[0, :3] = [5, 10**6, 7]
    out = torch.zeros((1, 16, 512), dtype=torch.bfloat16, device="cuda")
    ws = lib.workspace(lib.csa2_attn_workspace_size(1, 1))
    lib.csa2_sparse_attn_decode(dw.q[0], dw.kv, dev(idx), dev(np.array([3], np.int32)), 512,
                                dw.swa[0], dw.swa_len, 512 ** -0.5, out, ws)
    with pytest.raises(lib.Csa2Error) as e:
        lib.csa2_sync_status(ws)
    assert e.value.status == 7
    lib.csa2_sync_status(ws)  # cleared


def test_index_device_check_on_bad_page(lib, orc):
    """A page-table entry outside the row pool is never dereferenced by the
    scan (its TMA box is read as zeros), the rescore or the attention: the
    affected rows are skipped and csa2_sync_status reports
    CSA2_ERR_DEVICE_CHECK; the rest of the step still runs."""
    wl = synth.make("bp", seed=12, B=2, n_rows=[3000, 900], modes=[FULL], paged=True)
    dw = DeviceWorkload(lib, wl, orc)
    pt = wl.page_table.copy()
    pt[0, 5] = 10 ** 6          # page 5 of sequence 0: far outside the pool
    pt[1, 2] = -3               # a negative page id
    kv = lib.KVCache(dw.codes, dw.scales, dw.idxk, dw.n_rows, max_rows=int(wl.n_rows.max()),
                     page_table=dev(pt))
    idx = torch.full((2, 512), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((2,), -7, dtype=torch.int32, device="cuda")
    pool = torch.full((2, 2048), -7, dtype=torch.int32, device="cuda")
    pcnt = torch.full((2,), -7, dtype=torch.int32, device="cuda")
    ws = lib.workspace(lib.csa2_index_workspace_size(kv, 512, 2048))
    lib.csa2_index_full(kv, dw.q_idx[0], dw.w[0], 512, 2048, idx, cnt, pool, pcnt, ws)
    with pytest.raises(lib.Csa2Error) as e:
        lib.csa2_sync_status(ws)
    assert e.value.status == 7
    cnt = cnt.cpu().numpy()
    assert cnt[0] == 512 and cnt[1] == 512
    i0 = idx.cpu().numpy()
    assert not np.isin(i0[0], np.arange(5 * 64, 6 * 64)).any()   # nothing from the bad page
    assert not np.isin(i0[1], np.arange(2 * 64, 3 * 64)).any()
    lib.csa2_sync_status(ws)  # cleared


def test_host_side_argument_errors(lib, orc):
    wl = synth.make("at", seed=4, B=1, n_rows=[100], modes=[FULL])
    dw = DeviceWorkload(lib, wl, orc)
    ws = lib.workspace(16)
    idx = torch.zeros((1, 512), dtype=torch.int32, device="cuda")
    cnt = torch.zeros((1,), dtype=torch.int32, device="cuda")
    with pytest.raises(lib.Csa2Error) as e:      # workspace too small
        lib.csa2_index_full(dw.kv, dw.q_idx[0], dw.w[0], 512, 2048, idx, cnt,
                            torch.zeros((1, 2048), dtype=torch.int32, device="cuda"), cnt, ws)
    assert e.value.status == 4
    big = lib.workspace(1 << 20)
    with pytest.raises(lib.Csa2Error) as e:      # top_k out of range
        lib.csa2_index_full(dw.kv, dw.q_idx[0], dw.w[0], 513, 2048, idx, cnt,
                            torch.zeros((1, 2048), dtype=torch.int32, device="cuda"), cnt, big)
    assert e.value.status == 2
    with pytest.raises(lib.Csa2Error) as e:      # pool smaller than top_k
        lib.csa2_index_full(dw.kv, dw.q_idx[0], dw.w[0], 512, 100, idx, cnt,
                            torch.zeros((1, 2048), dtype=torch.int32, device="cuda"), cnt, big)
    assert e.value.status == 2
    with pytest.raises(lib.Csa2Error) as e:      # misaligned pointer
        lib.csa2_index_full(dw.kv, dw.q_idx[0], dw.w[0], 512, 2048,
                            torch.zeros(600, dtype=torch.int32, device="cuda")[1:513].view(1, 512),
                            cnt, torch.zeros((1, 2048), dtype=torch.int32, device="cuda"), cnt, big)
    assert e.value.status == 3
