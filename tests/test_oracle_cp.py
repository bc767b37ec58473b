"""Pins of the decomposition that context-parallel decode relies on, on the
oracle's own selection and attention (CPU):
  * the Top-k of the union of every shard's Top-k is the global Top-k, for any
    contiguous split, under the order (value desc, position asc), with many ties;
  * block maxima over shards whose boundaries are multiples of the block size
    are the global block maxima (and a boundary inside a block breaks this),
    so the pool from the concatenated shard maxima is the global pool;
  * attention over the union of two disjoint key sets is, per head, a convex
    combination of the attentions over each set (what the log-sum-exp merge of
    shard partials computes)."""
import numpy as np
import pytest

from fp4_kv_cache_quantize_b200 import synth


@pytest.mark.parametrize("seed", range(6))
def test_topk_of_shard_topks_is_the_global_topk(orc, seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 3000))
    if seed % 2:
        v = rng.integers(0, 7, n).astype(np.float64)  # heavy ties
    else:
        v = rng.standard_normal(n)
    k = int(rng.integers(1, 600))
    want = orc.select_topk(v, k)
    for world in (1, 2, 3, 5, 8):
        S = -(-n // world)
        union = []
        for r in range(world):
            lo, hi = r * S, min(n, (r + 1) * S)
            if hi <= lo:
                continue
            ids = np.arange(lo, hi, dtype=np.int64)
            union.append(orc.select_topk(v[lo:hi], k, ids=ids).astype(np.int64))
        u = np.concatenate(union) if union else np.zeros(0, np.int64)
        got = orc.select_topk(v[u], k, ids=u)
        assert np.array_equal(got, want), (seed, world)


def test_shard_topk_needs_the_position_tie_rule(orc):
    """With all values equal the global Top-k is the k lowest positions; a
    shard that kept its highest positions instead would lose them."""
    v = np.ones(64)
    want = orc.select_topk(v, 8)
    assert np.array_equal(want, np.arange(8))
    right = orc.select_topk(v[32:], 8, ids=np.arange(32, 64))
    assert np.array_equal(right, np.arange(32, 40))


def test_block_maxima_over_aligned_shards(orc):
    rng = np.random.default_rng(7)
    s = rng.standard_normal(5000)
    whole = orc.block_max(s, 8)
    for S in (128, 256, 1280):
        parts = [orc.block_max(s[lo:lo + S], 8) for lo in range(0, len(s), S)]
        assert np.array_equal(np.concatenate(parts), whole)
        assert np.array_equal(orc.pool(np.concatenate(parts), 64), orc.pool(whole, 64))
    # a shard boundary inside a block does not give the global maxima
    s2 = np.zeros(16)
    s2[5] = 1.0
    split = np.concatenate([orc.block_max(s2[:4], 8), orc.block_max(s2[4:], 8)])
    assert not np.array_equal(split, orc.block_max(s2, 8))


def test_attention_over_a_union_is_a_convex_combination(orc):
    wl = synth.make("cp_attn", seed=41, B=1, n_rows=[900], modes=[0], pool_blocks=0)
    x, k = wl.all_rows()
    codes, scales = orc.quantize_fp4(x)
    kv = orc.KV(codes, scales, k, seq_stride=wl.seq_stride)
    dm = orc.dims()
    rng = np.random.default_rng(3)
    sel = np.sort(rng.choice(900, 300, replace=False)).astype(np.int32)
    a, b = sel[:170], sel[170:]          # the two shards' rows
    sm = float(np.float32(512 ** -0.5))
    no_win = np.zeros((128, 512), np.uint8)
    q = wl.q[0, 0]
    o_ab = orc.attention(kv, dm, 0, q, sel, no_win, 0, sm)
    o_a = orc.attention(kv, dm, 0, q, a, no_win, 0, sm)
    o_b = orc.attention(kv, dm, 0, q, b, no_win, 0, sm)
    for h in range(dm.h):
        d, e = o_ab[h] - o_b[h], o_a[h] - o_b[h]
        lam = float(d @ e / (e @ e))
        assert 0.0 <= lam <= 1.0, (h, lam)
        assert np.linalg.norm(d - lam * e) <= 1e-9 * np.linalg.norm(e), h
    # and with the window on one side only (the rank that holds it)
    win = wl.swa[0, 0]
    o_aw = orc.attention(kv, dm, 0, q, a, win, 100, sm)
    o_all = orc.attention(kv, dm, 0, q, sel, win, 100, sm)
    for h in range(dm.h):
        d, e = o_all[h] - o_b[h], o_aw[h] - o_b[h]
        lam = float(d @ e / (e @ e))
        assert 0.0 <= lam <= 1.0 and np.linalg.norm(d - lam * e) <= 1e-9 * np.linalg.norm(e)
