"""Pins of the oracle's multi-query (draft verification) decode step.

Query t of a sequence must equal one single-query decode step on a cache and
a window that this test truncates physically (fresh arrays holding only the
entries query t may see), must not depend on anything a later draft added,
and with one query the step is the plain decode step."""
import numpy as np
import pytest

from fp4_kv_cache_quantize_b200 import synth

FULL, REINDEX, REUSE = 0, 1, 2


def _case(orc, Q, n_rows, swa_len, seed, paged=False):
    B = len(n_rows)
    L, modes = 3, [FULL, REINDEX, REUSE]
    wl = synth.make("mq", seed=seed, B=B, n_rows=n_rows, modes=modes, pool_blocks=32,
                    top_k=64, paged=paged)
    x, k = wl.all_rows()
    codes, scales = orc.quantize_fp4(x)
    kv = orc.KV(codes, scales, k, seq_stride=wl.seq_stride, page_table=wl.page_table)
    rng = np.random.default_rng(seed)
    bf = lambda a: synth.to_bf16_bits(np.asarray(a, np.float32))  # noqa: E731
    q_idx = bf(rng.standard_normal((L, B, Q, 8, 64)))
    w = rng.uniform(0, 1, (L, B, Q, 8)).astype(np.float32)
    q = bf(rng.standard_normal((L, B, Q, 16, 512)))
    swa = synth.to_e4m3_bits(rng.standard_normal((L, B, 128 + Q - 1, 512)).astype(np.float32))
    return dict(wl=wl, kv=kv, modes=modes, q_idx=q_idx, w=w, q=q, swa=swa,
                swa_len=np.asarray(swa_len, np.int32), L=L, B=B, Q=Q,
                n_rows=np.asarray(n_rows, np.int64), codes=codes, scales=scales, k=k)


def _run(orc, c, **over):
    a = dict(c, **over)
    return orc.layer_group_multi(a["kv"], orc.dims(), a["n_rows"], a["Q"], a["modes"],
                                 a["q_idx"], a["w"], a["q"], a["swa"], a["swa_len"], top_k=64,
                                 pool_blocks=32)


@pytest.mark.parametrize("paged", [False, True])
def test_each_query_is_a_decode_step_on_its_own_truncated_caches(orc, paged):
    c = _case(orc, 3, [700, 333], [130, 5], seed=21, paged=paged)
    got = _run(orc, c)
    for b in range(c["B"]):
        for t in range(c["Q"]):
            Ct = int(c["n_rows"][b]) - (c["Q"] - 1 - t)
            rows = np.array([c["kv"].row_of(b, p) for p in range(Ct)], np.int64)
            kv1 = orc.KV(c["codes"][rows], c["scales"][rows], c["k"][rows], seq_stride=max(Ct, 1))
            e = int(c["swa_len"][b]) - (c["Q"] - 1 - t)
            s0 = max(0, e - 128)
            win = np.zeros((c["L"], 1, 128, 512), np.uint8)
            win[:, 0, :e - s0] = c["swa"][:, b, s0:e]
            ref = orc.layer_group(kv1, orc.dims(), [Ct], c["modes"], c["q_idx"][:, b, t:t + 1],
                                  c["w"][:, b, t:t + 1], c["q"][:, b, t:t + 1], win, [e - s0],
                                  top_k=64, pool_blocks=32)
            assert np.array_equal(got["idx"][:, b, t], ref["idx"][:, 0]), (b, t)
            assert np.array_equal(got["idx_count"][:, b, t], ref["idx_count"][:, 0]), (b, t)
            assert np.array_equal(got["pool"][b, t], ref["pool"][0]), (b, t)
            assert np.array_equal(got["out"][:, b, t], ref["out"][:, 0]), (b, t)


def test_a_query_does_not_see_later_drafts(orc):
    c = _case(orc, 4, [500, 260], [131, 40], seed=22)
    base = _run(orc, c)
    # change what only the last draft of each sequence added
    codes, scales, k = c["codes"].copy(), c["scales"].copy(), c["k"].copy()
    swa = c["swa"].copy()
    for b in range(c["B"]):
        r = c["kv"].row_of(b, int(c["n_rows"][b]) - 1)
        codes[r] ^= 0x11
        k[r] ^= 0x0101
        swa[:, b, int(c["swa_len"][b]) - 1] ^= 0x21
    kv2 = orc.KV(codes, scales, k, seq_stride=c["wl"].seq_stride)
    other = _run(orc, c, kv=kv2, swa=swa)
    for key in ("idx", "out"):
        assert np.array_equal(base[key][:, :, :3], other[key][:, :, :3]), key
    assert not np.array_equal(base["out"][:, :, 3], other["out"][:, :, 3])


def test_one_query_is_the_plain_decode_step(orc):
    c = _case(orc, 1, [600, 90], [128, 17], seed=23)
    got = _run(orc, c)
    ref = orc.layer_group(c["kv"], orc.dims(), c["n_rows"], c["modes"], c["q_idx"][:, :, 0],
                          c["w"][:, :, 0], c["q"][:, :, 0], c["swa"], c["swa_len"], top_k=64,
                          pool_blocks=32)
    assert np.array_equal(got["idx"][:, :, 0], ref["idx"])
    assert np.array_equal(got["out"][:, :, 0], ref["out"])
