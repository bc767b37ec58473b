"""Pins of the oracle's cache-append step (the next row of work after the
decode path): the indexer-K projection against closed forms, hand-made
rounding ties and an independent nearest-bf16 property over numpy's fp64
matmul; the window ring against torch's E4M3 cast and its counter
invariants; the main-KV row placement for contiguous and paged layouts; and
the skip rule for positions without a row."""
import numpy as np
import pytest
import torch

from fp4_kv_cache_quantize_b200 import synth


def bf16_bits(a):
    return synth.to_bf16_bits(np.asarray(a, np.float32))


def bf16_vals(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def test_projection_of_a_one_hot_entry_is_one_rounded_row(orc):
    rng = np.random.default_rng(1)
    w = bf16_bits(rng.standard_normal((512, 64)) * 0.05)
    for c, a in [(0, 1.0), (17, -3.5), (511, 0.0078125)]:
        x = np.zeros(512, np.uint16)
        x[c] = bf16_bits([a])[0]
        got = orc.project_idxk(x, w)
        # a product of two bf16 values has at most 16 significant bits: it is
        # exact in fp32, so torch's single rounding to bf16 is the reference
        want = torch.from_numpy((a * bf16_vals(w[c])).astype(np.float32)).to(torch.bfloat16)
        assert np.array_equal(got, want.view(torch.int16).numpy().view(np.uint16)), c


def test_projection_rounding_ties_go_to_even(orc):
    w = np.zeros((512, 64), np.uint16)
    w[0, 0] = w[1, 0] = bf16_bits([1.0])[0]
    x = np.zeros(512, np.uint16)
    x[0] = bf16_bits([1.0])[0]
    x[1] = bf16_bits([2.0 ** -8])[0]          # 1 + 2^-8: midway between 1 and 1 + 2^-7
    assert orc.project_idxk(x, w)[0] == 0x3F80
    x[1] = bf16_bits([3 * 2.0 ** -8])[0]      # midway between 1 + 2^-7 and 1 + 2^-6
    assert orc.project_idxk(x, w)[0] == 0x3F82
    x[1] = bf16_bits([-(2.0 ** -8)])[0]       # 1 - 2^-8 is a bf16 value: exact
    assert orc.project_idxk(x, w)[0] == bf16_bits([1 - 2.0 ** -8])[0]


def test_synthetic_indexer_k_rounds_once_like_the_append_rule(orc):
    """The decode inputs' indexer K (synth) follows the append path's rule:
    the fp64 sum rounded once to bf16.  Sums that sit on a bf16 rounding
    midpoint in fp64 but not after a float32 step tell one rounding from two."""
    w = np.zeros((512, 64), np.uint16)
    w[0, :] = bf16_bits([1.0])[0]
    w[1, :] = bf16_bits([2.0 ** -8])[0]
    w[2, :] = bf16_bits([2.0 ** -30])[0]
    x = np.zeros((6, 512), np.uint16)
    x[:, 0] = bf16_bits([1.0])[0]
    x[0, 1] = bf16_bits([1.0])[0]                      # 1 + 2^-8: tie, to even (1)
    x[1, 1], x[1, 2] = bf16_bits([1.0])[0], bf16_bits([1.0])[0]   # just above the tie
    x[2, 1], x[2, 2] = bf16_bits([1.0])[0], bf16_bits([-1.0])[0]  # just below the tie
    x[3, 1] = bf16_bits([3.0])[0]                      # 1 + 3 2^-8: tie, to even (1 + 2^-6)
    x[4, 2] = bf16_bits([5.0])[0]                      # 1 + 5 2^-30: rounds to 1
    x[5] = bf16_bits(np.random.default_rng(3).standard_normal(512))
    wl = type("W", (), {"w_idx": w})()
    got = synth.Workload.idxk_of(wl, x)
    want = np.stack([orc.project_idxk(x[i], w) for i in range(len(x))])
    assert np.array_equal(got, want)
    # the float32 step would have moved the first "just above" and "just
    # below" sums onto the tie (1 + 2^-8 +- 2^-30 is not a float32 value)
    assert got[1, 0] == 0x3F81 and got[2, 0] == 0x3F80
    assert not np.array_equal(got, synth.to_bf16_bits(
        (bf16_vals(x) @ bf16_vals(w)).astype(np.float32)))


def _neighbours(bits):
    return (bits.astype(np.int32) + 1).astype(np.uint16), (bits.astype(np.int32) - 1).astype(np.uint16)


def test_projection_is_the_nearest_bf16_to_the_exact_sum(orc):
    rng = np.random.default_rng(2)
    w = bf16_bits(rng.standard_normal((512, 64)) / np.sqrt(512))
    for trial in range(6):
        x = bf16_bits(rng.standard_normal(512) * (10.0 ** (trial - 2)))
        got = orc.project_idxk(x, w)
        v = bf16_vals(x) @ bf16_vals(w)                # fp64 sums of exact products
        g = bf16_vals(got)
        up, dn = _neighbours(got)
        assert np.all(np.sign(g) * np.sign(v) >= 0)
        assert np.all(np.abs(g - v) <= np.abs(bf16_vals(up) - v))
        assert np.all(np.abs(g - v) <= np.abs(bf16_vals(dn) - v))


def _kv(orc, rows, seq_stride=0, page_table=None):
    return orc.KV(np.zeros((rows, 256), np.uint8), np.zeros((rows, 32), np.uint8),
                  np.zeros((rows, 64), np.uint16), seq_stride=seq_stride, page_table=page_table)


@pytest.mark.parametrize("paged", [False, True])
def test_main_rows_land_at_the_mapped_row_and_counters_advance(orc, paged):
    rng = np.random.default_rng(3)
    B = 3
    if paged:
        pt = np.array([[5, 2, -1], [0, 7, 3], [1, 4, 6]], np.int32)
        kv = _kv(orc, 8 * 64, page_table=pt)
        n_rows = np.array([63, 64, 130], np.int64)
    else:
        kv = _kv(orc, 3 * 200, seq_stride=200)
        n_rows = np.array([0, 57, 199], np.int64)
    dm = orc.dims()
    w = bf16_bits(rng.standard_normal((512, 64)) / np.sqrt(512))
    x = bf16_bits(rng.standard_normal((B, 512)))
    start = n_rows.copy()
    assert orc.cache_append(kv, dm, n_rows, x, w) == 0
    assert np.array_equal(n_rows, start + 1)
    for b in range(B):
        row = kv.row_of(b, int(start[b]))
        want_row = (pt[b, start[b] // 64] * 64 + start[b] % 64) if paged else b * 200 + start[b]
        assert row == want_row
        codes, scales = orc.quantize_fp4(x[b:b + 1])
        assert np.array_equal(kv.codes[row], codes[0]) and np.array_equal(kv.scales[row], scales[0])
        assert np.array_equal(kv.idxk[row], orc.project_idxk(x[b], w))
        others = np.ones(kv.codes.shape[0], bool)
        others[[kv.row_of(bb, int(start[bb])) for bb in range(B)]] = False
        assert not kv.codes[others].any() and not kv.idxk[others].any()


def test_positions_without_a_row_are_skipped(orc):
    dm = orc.dims()
    w = np.zeros((512, 64), np.uint16)
    x = bf16_bits(np.ones((2, 512)))
    kv = _kv(orc, 2 * 100, seq_stride=100)
    n_rows = np.array([100, 5], np.int64)          # sequence 0 is full
    assert orc.cache_append(kv, dm, n_rows, x, w) == 1
    assert n_rows.tolist() == [100, 6]
    assert not kv.codes[:100].any() and kv.codes[105].any()
    pt = np.array([[3, -1]], np.int32)
    kv = _kv(orc, 4 * 64, page_table=pt)
    n_rows = np.array([64], np.int64)               # page 1 is not mapped
    assert orc.cache_append(kv, dm, n_rows, x[:1], w) == 1
    assert n_rows.tolist() == [64] and not kv.codes.any()


def test_window_ring_holds_the_last_w_entries(orc):
    rng = np.random.default_rng(4)
    dm = orc.dims()
    B, L, W = 2, 3, 128
    kv = _kv(orc, 2 * 400, seq_stride=400)
    n_rows = np.array([0, 10], np.int64)
    w = np.zeros((512, 64), np.uint16)
    swa = np.zeros((L, B, W, 512), np.uint8)
    swa_pos = np.array([0, 70], np.int64)
    swa_len = np.zeros(B, np.int32)
    history = {b: [] for b in range(B)}
    for step in range(140):
        x = bf16_bits(rng.standard_normal((B, 512)))
        xs = bf16_bits(rng.standard_normal((L, B, 512)) * 4)
        pos_before = swa_pos.copy()
        assert orc.cache_append(kv, dm, n_rows, x, w, xs, swa, swa_pos, swa_len) == 0
        assert np.array_equal(swa_pos, pos_before + 1)
        assert np.array_equal(swa_len, np.minimum(swa_pos, W))
        for b in range(B):
            history[b].append((int(pos_before[b]), xs[:, b]))
    for b in range(B):
        for pos, xs_b in history[b][-W:]:
            want = torch.from_numpy(bf16_vals(xs_b).astype(np.float32)).to(torch.float8_e4m3fn)
            assert np.array_equal(swa[:, b, pos % W], want.view(torch.uint8).numpy()), (b, pos)


def test_window_entries_saturate_instead_of_overflowing(orc):
    dm = orc.dims()
    kv = _kv(orc, 64, seq_stride=64)
    n_rows = np.array([0], np.int64)
    xs = bf16_bits(np.array([[[1e4] * 256 + [-1e4] * 256]]))
    swa = np.zeros((1, 1, 128, 512), np.uint8)
    pos = np.array([5], np.int64)
    ln = np.zeros(1, np.int32)
    orc.cache_append(kv, dm, n_rows, bf16_bits(np.zeros((1, 512))), np.zeros((512, 64), np.uint16),
                     xs, swa, pos, ln)
    assert (swa[0, 0, 5, :256] == 0x7E).all() and (swa[0, 0, 5, 256:] == 0xFE).all()
    assert ln.tolist() == [6] and pos.tolist() == [6]
