"""Pins of the oracle's indexer (scores, block maxima, HSI pool, Top-K,
Reindex, Reuse) and of its attention, each against something other than the
oracle itself: closed forms, brute force with Python's sort or numpy, and the
invariants the pages fix (Reuse copies indices, Reindex stays in the pool,
the Full Top-K lies inside the pool, paging does not change results).
"""
import numpy as np
import pytest
import torch

from fp4_kv_cache_quantize_b200 import synth

FULL, REINDEX, REUSE = 0, 1, 2


def bf16(a):
    return torch.tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def f_of(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def brute_topk(v, k, ids=None):
    ids = np.arange(len(v)) if ids is None else np.asarray(ids)
    order = sorted(range(len(v)), key=lambda i: (-v[i], ids[i]))
    return np.sort(ids[order[:k]])


# ------------------------------------------------------------------ scores
def test_scores_closed_form_unit_keys(orc):
    dm = orc.dims(d=32, h=2, hi=8, di=64, blk=8, w=4)
    C = 128
    k = np.zeros((C, 64), np.float32)
    k[np.arange(C), np.arange(C) % 64] = 1.0 + (np.arange(C) // 64)      # 1 or 2
    q = np.array([[((h * 7 + d * 3) % 11) - 5 for d in range(64)] for h in range(8)], np.float32)
    w = (np.arange(8, dtype=np.float32) + 1) / 8
    kv = orc.KV(np.zeros((C, 16), np.uint8), np.zeros((C, 2), np.uint8), bf16(k), seq_stride=C)
    s = orc.scores(kv, dm, 0, C, bf16(q), w)
    for p in range(C):
        mag = 1.0 + p // 64
        want = sum(float(w[h]) * max(0.0, q[h, p % 64] * mag) for h in range(8))
        assert s[p] == want


def test_scores_match_numpy_fp64(orc):
    g = np.random.default_rng(5)
    dm = orc.dims()
    C = 300
    k = bf16(g.standard_normal((C, 64)))
    q = bf16(g.standard_normal((8, 64)))
    w = g.random(8).astype(np.float32)
    kv = orc.KV(np.zeros((C, 256), np.uint8), np.zeros((C, 32), np.uint8), k, seq_stride=C)
    s = orc.scores(kv, dm, 0, C, q, w)
    want = np.maximum(f_of(q) @ f_of(k).T, 0).T @ w.astype(np.float64)
    np.testing.assert_allclose(s, want, rtol=1e-13, atol=1e-12)


# ------------------------------------------------------- selection / pool
@pytest.mark.parametrize("n,k", [(1, 1), (7, 3), (64, 64), (100, 7), (513, 512), (40, 100)])
def test_select_topk_brute_force_with_ties(orc, n, k):
    g = np.random.default_rng(n * 31 + k)
    for _ in range(20):
        v = g.integers(0, 5, n).astype(np.float64)          # many ties
        got = orc.select_topk(v, k)
        assert np.array_equal(got, brute_topk(v, k))
        ids = g.permutation(10 * n)[:n]
        assert np.array_equal(orc.select_topk(v, k, ids), brute_topk(v, k, ids))


def test_block_max_brute_force(orc):
    g = np.random.default_rng(6)
    for C in (1, 7, 8, 9, 63, 64, 65):
        s = g.integers(-3, 4, C).astype(np.float64)
        bm = orc.block_max(s, 8)
        assert len(bm) == (C + 7) // 8
        for j in range(len(bm)):
            assert bm[j] == max(s[8 * j:8 * j + 8])


def test_pool_counts_and_order(orc):
    g = np.random.default_rng(7)
    for nblk, pb in ((5, 2048), (2048, 2048), (3000, 2048), (10, 3)):
        bm = g.integers(0, 6, nblk).astype(np.float64)
        p = orc.pool(bm, pb)
        assert len(p) == min(pb, nblk)
        assert np.all(np.diff(p) > 0)
        assert np.array_equal(p, brute_topk(bm, pb))


def test_full_topk_lies_inside_pool_theorem(orc):
    """Top-k positions lie in the top-k blocks by block max when ties break
    to the lower position / lower block id.  Integer scores, many ties."""
    g = np.random.default_rng(8)
    for trial in range(300):
        C = int(g.integers(1, 200))
        k = int(g.integers(1, 40))
        s = g.integers(0, 4, C).astype(np.float64)
        top = orc.select_topk(s, k)
        pool = orc.pool(orc.block_max(s, 8), k)
        assert set((top // 8).tolist()) <= set(pool.tolist()), trial


# ------------------------------------------------------------ layer group
def small_wl(B=2, n_rows=(200, 77), modes=(FULL, REUSE, REINDEX, REUSE), paged=False,
             pool_blocks=6, top_k=16, seed=11):
    return synth.make("t", seed=seed, B=B, n_rows=list(n_rows), modes=list(modes),
                      top_k=top_k, pool_blocks=pool_blocks, paged=paged,
                      d=32, h=2, hi=3, di=16, blk=8, w=4, swa_len=[4] * B)


def run_group(orc, wl):
    x, k = wl.all_rows()
    codes, scales = orc.quantize_fp4(x)
    kv = orc.KV(codes, scales, k, seq_stride=wl.seq_stride, page_table=wl.page_table)
    dm = orc.dims(d=wl.d, h=wl.h, hi=wl.hi, di=wl.di, blk=wl.blk, w=wl.w)
    r = orc.layer_group(kv, dm, wl.n_rows, wl.modes, wl.q_idx, wl.w_h, wl.q, wl.swa,
                        wl.swa_len, top_k=wl.top_k, pool_blocks=wl.pool_blocks)
    return r, kv, dm, codes, scales


def test_group_modes_reuse_reindex_and_full(orc):
    wl = small_wl()
    r, kv, dm, _, _ = run_group(orc, wl)
    for b in range(wl.B):
        C = int(wl.n_rows[b])
        # Full: the exact top-k over all visible positions
        s0 = orc.scores(kv, dm, b, C, wl.q_idx[0, b], wl.w_h[0, b])
        assert np.array_equal(r["idx"][0, b, :r["idx_count"][0, b]], brute_topk(s0, wl.top_k))
        # pool: top blocks of the Full layer's block maxima
        bm = [max(s0[8 * j:8 * j + 8]) for j in range((C + 7) // 8)]
        pool = r["pool"][b, :r["pool_count"][b]]
        assert np.array_equal(pool, brute_topk(np.array(bm), wl.pool_blocks))
        # Reuse: byte-identical to the latest indices
        assert np.array_equal(r["idx"][1, b], r["idx"][0, b])
        assert np.array_equal(r["idx"][3, b], r["idx"][2, b])
        # Reindex: own query, only positions inside the pool
        picks = r["idx"][2, b, :r["idx_count"][2, b]]
        assert set((picks // 8).tolist()) <= set(pool.tolist())
        cand = np.array([p for j in pool for p in range(8 * j, min(8 * j + 8, C))])
        s2 = orc.scores(kv, dm, b, C, wl.q_idx[2, b], wl.w_h[2, b])
        assert np.array_equal(picks, brute_topk(s2[cand], wl.top_k, cand))


def test_group_without_pool_reindex_sees_everything(orc):
    wl = small_wl(modes=(FULL, REINDEX), pool_blocks=0)
    r, kv, dm, _, _ = run_group(orc, wl)
    for b in range(wl.B):
        C = int(wl.n_rows[b])
        s1 = orc.scores(kv, dm, b, C, wl.q_idx[1, b], wl.w_h[1, b])
        assert np.array_equal(r["idx"][1, b, :r["idx_count"][1, b]], brute_topk(s1, wl.top_k))
    assert np.all(r["pool_count"] == 0)


def test_group_paged_equals_contiguous(orc):
    """Same per-sequence rows through a shuffled page table: same results."""
    wl_c = small_wl(n_rows=(150, 64))
    r_c, kv_c, dm, codes, scales = run_group(orc, wl_c)
    x, k = wl_c.all_rows()
    # build a paged pool holding the same rows, pages shuffled
    B = wl_c.B
    pages = [(int(c) + 63) // 64 for c in wl_c.n_rows]
    perm = np.random.default_rng(12).permutation(sum(pages))
    pt = np.zeros((B, max(pages)), np.int32)
    codes_p = np.zeros((sum(pages) * 64, codes.shape[1]), np.uint8)
    scales_p = np.zeros((sum(pages) * 64, scales.shape[1]), np.uint8)
    k_p = np.zeros((sum(pages) * 64, k.shape[1]), np.uint16)
    off = 0
    for b in range(B):
        for j in range(pages[b]):
            pid = perm[off + j]
            pt[b, j] = pid
            src = slice(b * wl_c.seq_stride + 64 * j, b * wl_c.seq_stride + 64 * j + 64)
            dst = slice(64 * pid, 64 * pid + 64)
            codes_p[dst], scales_p[dst], k_p[dst] = codes[src], scales[src], k[src]
        off += pages[b]
    kv_p = orc.KV(codes_p, scales_p, k_p, page_table=pt)
    r_p = orc.layer_group(kv_p, dm, wl_c.n_rows, wl_c.modes, wl_c.q_idx, wl_c.w_h, wl_c.q,
                          wl_c.swa, wl_c.swa_len, top_k=wl_c.top_k, pool_blocks=wl_c.pool_blocks)
    for key in ("idx", "idx_count", "pool", "pool_count", "out"):
        assert np.array_equal(r_p[key], r_c[key]), key


def test_group_rejects_leading_reuse(orc):
    wl = small_wl(modes=(REUSE, FULL))
    with pytest.raises(ValueError):
        run_group(orc, wl)


# -------------------------------------------------------------- attention
def dense_attention(q_bits, rows, scale):
    qf = f_of(q_bits)
    lg = qf @ rows.T * scale
    lg -= lg.max(axis=1, keepdims=True)
    p = np.exp(lg)
    p /= p.sum(axis=1, keepdims=True)
    return p @ rows


def test_attention_is_dense_attention_when_all_selected(orc):
    """C <= top_k: the sparse branch selects every position, so the output is
    plain dense softmax attention over [all main-KV rows ; SWA rows]."""
    wl = small_wl(n_rows=(12, 5), modes=(FULL, REUSE), top_k=16)
    r, kv, dm, codes, scales = run_group(orc, wl)
    for b in range(wl.B):
        C = int(wl.n_rows[b])
        assert r["idx_count"][0, b] == C
        rows_main = orc.dequantize_fp4(codes[b * wl.seq_stride: b * wl.seq_stride + C],
                                       scales[b * wl.seq_stride: b * wl.seq_stride + C])
        for l in range(wl.L):
            swa = torch.tensor(wl.swa[l, b]).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
            rows = np.concatenate([rows_main, swa[: wl.swa_len[b]]])
            want = dense_attention(wl.q[l, b], rows, 1 / np.sqrt(wl.d))
            np.testing.assert_allclose(r["out"][l, b], want, rtol=1e-10, atol=1e-12)


def test_attention_single_key_and_uniform_logits(orc):
    g = np.random.default_rng(13)
    dm = orc.dims(d=32, h=2, hi=2, di=16, blk=8, w=4)
    x = bf16(g.standard_normal((10, 32)))
    codes, scales = orc.quantize_fp4(x)
    kv = orc.KV(codes, scales, np.zeros((10, 16), np.uint16), seq_stride=10)
    rows = orc.dequantize_fp4(codes, scales)
    q = bf16(g.standard_normal((2, 32)))
    swa = np.zeros((4, 32), np.uint8)
    out = orc.attention(kv, dm, 0, q, np.array([6], np.int32), swa, 0, 0.17)
    assert np.array_equal(out, np.stack([rows[6], rows[6]]))
    # zero query: every logit equal -> the mean of the rows
    out = orc.attention(kv, dm, 0, np.zeros((2, 32), np.uint16), np.array([1, 4, 9], np.int32),
                        swa, 0, 0.17)
    np.testing.assert_allclose(out[0], rows[[1, 4, 9]].mean(axis=0), rtol=1e-14, atol=1e-15)
    # nothing to attend to -> zeros
    out = orc.attention(kv, dm, 0, q, np.zeros(0, np.int32), swa, 0, 0.17)
    assert np.all(out == 0)
