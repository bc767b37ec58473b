"""GPU parity of csa2_layer_group (the whole decode step of a CSA2 layer group)
against the oracle's layer group: indices of every layer, the HSI pool, and
the attention output of every layer."""
import numpy as np
import pytest
import torch

from fp4_kv_cache_quantize_b200 import synth
from gpu_helpers import ATTN_RTOL, DeviceWorkload, bf16_to_f64, check_selection, rel_l2

pytestmark = pytest.mark.gpu
FULL, REINDEX, REUSE = 0, 1, 2


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp4_kv_cache_quantize_b200 import csa2
    return csa2


def run_group(lib, dw):
    wl = dw.wl
    grp = lib.LayerGroup(dw.kv, wl.modes, dw.q_idx, dw.w, dw.q, dw.swa, dw.swa_len,
                         top_k=wl.top_k, pool_blocks=wl.pool_blocks)
    ws = lib.workspace(grp.workspace_size())
    lib.csa2_layer_group(grp, ws)
    lib.csa2_sync_status(ws)
    return grp


def compare_group(orc, dw, grp, *, check_out=True, kv=None, ref=None):
    """kv/ref: the oracle's cache view and its layer-group result when the
    caller built them (full-size runs); else both come from dw."""
    wl = dw.wl
    kv = kv if kv is not None else dw.oracle_kv(orc)
    dm = orc.dims()
    if ref is None:
        ref = orc.layer_group(kv, dm, wl.n_rows, wl.modes, wl.q_idx, wl.w_h, wl.q, wl.swa,
                              wl.swa_len, top_k=wl.top_k, pool_blocks=wl.pool_blocks,
                              sm_scale=float(np.float32(512 ** -0.5)))
    idx = grp.idx.cpu().numpy()
    cnt = grp.idx_count.cpu().numpy()
    out = bf16_to_f64(grp.out)
    n_diff = 0
    for b in range(wl.B):
        C = int(wl.n_rows[b])
        s_full = None
        pool_ok = None
        for l in range(wl.L):
            m = wl.modes[l]
            if m == FULL:
                s_full = orc.scores(kv, dm, b, C, wl.q_idx[l, b], wl.w_h[l, b])
                s_l, cand = s_full, np.arange(C)
                if wl.pool_blocks:
                    bm = orc.block_max(s_full, 8)
                    gp = grp.pool.cpu().numpy()[b]
                    gpc = int(grp.pool_count.cpu().numpy()[b])
                    check_selection(gp, gpc, ref["pool"][b, :ref["pool_count"][b]],
                                    lambda j: bm[j], wl.pool_blocks,
                                    cand_positions=np.arange(len(bm)), what=f"pool b={b}")
                    thr = np.sort(bm)[::-1][min(wl.pool_blocks, len(bm)) - 1] if len(bm) else 0
                    pool_ok = lambda pos: np.abs(bm[pos // 8] - thr) <= 1e-5 * abs(thr)
            elif m == REINDEX:
                s_l = orc.scores(kv, dm, b, C, wl.q_idx[l, b], wl.w_h[l, b])
                if wl.pool_blocks:
                    op = ref["pool"][b, :ref["pool_count"][b]]
                    cand = np.array([p for j in op for p in range(8 * j, min(8 * j + 8, C))],
                                    dtype=np.int64)
                else:
                    cand = np.arange(C)
            want = ref["idx"][l, b, :ref["idx_count"][l, b]]
            n_diff += check_selection(idx[l, b], int(cnt[l, b]), want, lambda p: s_l[p],
                                      wl.top_k, cand_positions=cand,
                                      extra_ok=pool_ok if m == REINDEX else None,
                                      what=f"layer {l} b={b}")
            if m == REUSE:
                src = max(i for i in range(l) if wl.modes[i] != REUSE)
                assert np.array_equal(idx[l, b], idx[src, b]) and cnt[l, b] == cnt[src, b]
            if check_out:
                err = rel_l2(out[l, b], ref["out"][l, b])
                assert err <= ATTN_RTOL, (l, b, err)
    return n_diff


def test_group_tiny_config(lib, orc):
    """The tiny workload: batch 1, context 4,096, Full + 3 Reuse."""
    wl = synth.config(0)
    dw = DeviceWorkload(lib, wl, orc)
    compare_group(orc, dw, run_group(lib, dw))


def test_group_hsi_reduced(lib, orc):
    """Decoder HSI group (Full, Reindex, 3 Reuse) at a reduced context with a
    real 2,048-block pool and ragged lengths."""
    wl = synth.make("hsi", seed=77, B=3, n_rows=[40000, 16500, 5],
                    modes=[FULL, REINDEX, REUSE, REUSE, REUSE])
    dw = DeviceWorkload(lib, wl, orc)
    compare_group(orc, dw, run_group(lib, dw))


def test_group_decoder_pattern_reduced(lib, orc):
    """The 20-layer decoder pattern with planted blocks, reduced context."""
    wl = synth.make("dec", seed=78, B=1, n_rows=[50000], modes=synth.DECODER_20,
                    planted_blocks=64)
    dw = DeviceWorkload(lib, wl, orc)
    compare_group(orc, dw, run_group(lib, dw))


def test_group_ragged_paged_no_pool(lib, orc):
    """Encoder-style group (Full + 5 Reuse, no pool) over a shuffled page
    pool, ragged lengths."""
    g = np.random.default_rng(5)
    n_rows = g.integers(100, 9000, size=6)
    wl = synth.make("pg", seed=79, B=6, n_rows=n_rows, modes=[FULL] + [REUSE] * 5,
                    pool_blocks=0, paged=True)
    dw = DeviceWorkload(lib, wl, orc)
    compare_group(orc, dw, run_group(lib, dw))


def test_group_query_magnitudes(lib, orc):
    """Main queries whose heads span bf16's range, from 1e-6 to 1e5 (beyond
    fp16's 65,504) and all-zero heads: the attention must match the oracle
    with no overflow and no loss of small queries."""
    wl = synth.config(0)
    q = synth.bf16_bits_to_f32(wl.q).astype(np.float64)
    scale = np.array([1e-6, 3e-5, 1e-3, 0.25, 1.0, 7.0, 100.0, 2e3,
                      3e4, 6.5e4, 1e5, 1e5, 0.0, 1.0, 1e-6, 5e4])
    for l in range(wl.L):
        sc = np.roll(scale, l)
        q[l] *= sc[None, :, None]
    wl.q = synth.to_bf16_bits(q.astype(np.float32))
    assert np.abs(synth.bf16_bits_to_f32(wl.q)).max() > 65504.0
    dw = DeviceWorkload(lib, wl, orc)
    compare_group(orc, dw, run_group(lib, dw))


def test_group_rejects_leading_reuse(lib, orc):
    wl = synth.make("bad", seed=3, B=1, n_rows=[100], modes=[REUSE, FULL])
    dw = DeviceWorkload(lib, wl, orc)
    with pytest.raises(lib.Csa2Error) as e:
        run_group(lib, dw)
    assert e.value.status == 1
