"""GPU parity of the context-parallel decode step (csa2_cp_* entry points,
driven by fp4_kv_cache_quantize_b200.cp) with every shard run on one device
through LocalComm.  For 1 to 4 shards, contiguous and paged caches, with and
without the HSI pool:
  * every shard's indices and pool equal the one-device csa2_layer_group's
    exactly (the shards exchange keys bit-identical to the ones the
    one-device rescore ranks, and the merge keeps its tie rule);
  * indices, pool and attention output match the oracle's layer group under
    the usual tolerances (ties within 1e-5; attention relative L2 <= 5e-3).
"""
import numpy as np
import pytest
import torch

from fp4_kv_cache_quantize_b200 import synth
from gpu_helpers import ATTN_RTOL, DeviceWorkload, bf16_to_f64, rel_l2
from test_gpu_group import compare_group

pytestmark = pytest.mark.gpu
FULL, REINDEX, REUSE = 0, 1, 2


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp4_kv_cache_quantize_b200 import csa2
    return csa2


def relayout(dw, stride):
    """The workload's cache with sequence b at rows [b * stride, ...)."""
    wl = dw.wl
    rows = wl.B * stride
    codes = torch.zeros((rows, 256), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((rows, 32), dtype=torch.uint8, device="cuda")
    idxk = torch.zeros((rows, 64), dtype=torch.int16, device="cuda")
    for b in range(wl.B):
        n = int(wl.n_rows[b])
        src = torch.from_numpy(wl.row_of(b, np.arange(n))).cuda()
        codes[b * stride:b * stride + n] = dw.codes[src]
        scales[b * stride:b * stride + n] = dw.scales[src]
        idxk[b * stride:b * stride + n] = dw.idxk[src]
    return codes, scales, idxk


def run_cp(lib, dw, world, *, paged):
    from fp4_kv_cache_quantize_b200 import cp
    wl = dw.wl
    S = cp.shard_rows_for(int(wl.n_rows.max()), world)
    if paged:
        codes, scales, idxk, stride, pt = dw.codes, dw.scales, dw.idxk, 0, dw.page_table
    else:
        stride = world * S
        codes, scales, idxk = relayout(dw, stride)
        pt = None
    ranks = []
    for r in range(world):
        kv = cp.local_view(codes, scales, idxk, rank=r, world=world, shard_rows=S, batch=wl.B,
                           seq_stride=stride, page_table=pt)
        ranks.append(cp.CPRank(kv, rank=r, world=world, shard_rows=S, n_layers=wl.L,
                               top_k=wl.top_k, pool_blocks=wl.pool_blocks))
    cp.cp_layer_group(ranks, cp.LocalComm(world), wl.modes, dw.n_rows, dw.q_idx, dw.w, dw.q,
                      dw.swa, dw.swa_len, sm_scale=float(np.float32(512 ** -0.5)))
    for r in ranks:
        lib.csa2_sync_status(r.ws)
    return ranks


def one_device(lib, dw):
    wl = dw.wl
    grp = lib.LayerGroup(dw.kv, wl.modes, dw.q_idx, dw.w, dw.q, dw.swa, dw.swa_len,
                         top_k=wl.top_k, pool_blocks=wl.pool_blocks,
                         sm_scale=float(np.float32(512 ** -0.5)))
    ws = lib.workspace(grp.workspace_size())
    lib.csa2_layer_group(grp, ws)
    lib.csa2_sync_status(ws)
    return grp


def check(lib, orc, wl, world, paged):
    dw = DeviceWorkload(lib, wl, orc)
    ranks = run_cp(lib, dw, world, paged=paged)
    grp = one_device(lib, dw)
    for r in ranks:
        assert torch.equal(r.idx_count, grp.idx_count), r.shard.rank
        for l in range(wl.L):
            for b in range(wl.B):
                n = int(grp.idx_count[l, b])
                assert torch.equal(r.idx[l, b], grp.idx[l, b]), (r.shard.rank, l, b, n)
        if wl.pool_blocks:
            assert torch.equal(r.pool_count, grp.pool_count)
            assert torch.equal(r.pool, grp.pool)
        # the shards' outputs agree with the one-device step to bf16 rounding
        err = rel_l2(bf16_to_f64(r.out), bf16_to_f64(grp.out))
        assert err <= ATTN_RTOL, (r.shard.rank, err)
    compare_group(orc, dw, ranks[0])
    compare_group(orc, dw, ranks[-1])


@pytest.mark.parametrize("world", [1, 2, 3, 4])
def test_cp_contiguous_hsi_group(lib, orc, world):
    wl = synth.make("cp", seed=500 + world, B=2, n_rows=[20000, 300],
                    modes=[FULL, REUSE, REINDEX, REUSE, FULL, REINDEX], pool_blocks=2048,
                    swa_len=[128, 37])
    check(lib, orc, wl, world, paged=False)


@pytest.mark.parametrize("world", [2, 3])
def test_cp_paged_without_pool(lib, orc, world):
    wl = synth.make("cp", seed=520 + world, B=3, n_rows=[9000, 4099, 64],
                    modes=[FULL, REINDEX, REUSE], pool_blocks=0, paged=True,
                    swa_len=[128, 0, 5])
    check(lib, orc, wl, world, paged=True)


def test_cp_query_magnitudes(lib, orc):
    """Shards attend with the split-KV kernel: main queries whose heads span
    bf16's range (1e-6 to 1e5, beyond fp16's 65,504, and all-zero heads)
    must match the oracle with no overflow and no loss of small queries."""
    wl = synth.make("cp", seed=540, B=2, n_rows=[6000, 900],
                    modes=[FULL, REUSE, REINDEX], pool_blocks=2048, swa_len=[128, 60])
    q = synth.bf16_bits_to_f32(wl.q).astype(np.float64)
    scale = np.array([1e-6, 3e-5, 1e-3, 0.25, 1.0, 7.0, 100.0, 2e3,
                      3e4, 6.5e4, 1e5, 1e5, 0.0, 1.0, 1e-6, 5e4])
    for l in range(wl.L):
        q[l] *= np.roll(scale, 3 * l)[None, :, None]
    wl.q = synth.to_bf16_bits(q.astype(np.float32))
    assert np.abs(synth.bf16_bits_to_f32(wl.q)).max() > 65504.0
    check(lib, orc, wl, 2, paged=False)


def test_cp_attention_only_window(lib, orc):
    """A sequence with no global entries: every shard's rows are empty and
    the output is the window-only attention of the rank holding the window."""
    wl = synth.make("cp", seed=530, B=2, n_rows=[0, 700], modes=[FULL, REUSE],
                    pool_blocks=0, swa_len=[90, 128])
    dw = DeviceWorkload(lib, wl, orc)
    ranks = run_cp(lib, dw, 2, paged=False)
    kv = dw.oracle_kv(orc)
    ref = orc.layer_group(kv, orc.dims(), wl.n_rows, wl.modes, wl.q_idx, wl.w_h, wl.q, wl.swa,
                          wl.swa_len, top_k=wl.top_k, pool_blocks=0,
                          sm_scale=float(np.float32(512 ** -0.5)))
    out = bf16_to_f64(ranks[1].out)
    for l in range(wl.L):
        for b in range(wl.B):
            assert rel_l2(out[l, b], ref["out"][l, b]) <= ATTN_RTOL, (l, b)
    assert int(ranks[0].idx_count[0, 0]) == 0


def test_cp_rejects_bad_shards(lib):
    from fp4_kv_cache_quantize_b200 import cp
    assert lib.csa2_cp_workspace_size(lib.CpShard(0, 2, 100), 1, 1, 512) == 0  # not x128
    assert lib.csa2_cp_workspace_size(lib.CpShard(2, 2, 128), 1, 1, 512) == 0  # rank >= world
    assert lib.csa2_cp_workspace_size(lib.CpShard(0, 17, 128), 1, 1, 512) == 0  # world > 16
    assert lib.csa2_cp_workspace_size(lib.CpShard(0, 2, 1 << 20), 1, 1, 512) == 0  # > 1M rows
    assert cp.shard_rows_for(20000, 3) == 6784
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(lib.Csa2Error) as e:
        lib.csa2_cp_filter(lib.CpShard(0, 2, 128), 3, n.view(1, 1), n, n.view(1, 1), n,
                           lib.workspace(256))
    assert e.value.status == 1


def test_cp_batched_calls_equal_single_calls(lib, orc):
    """The batched entry points (all jobs of a pool, every layer's filter in
    one launch) give bit-identical results to the per-job / per-layer calls."""
    wl = synth.make("cp", seed=560, B=2, n_rows=[20000, 3000],
                    modes=[FULL, REUSE, REINDEX, REUSE, FULL, REINDEX], pool_blocks=2048,
                    swa_len=[128, 37])
    dw = DeviceWorkload(lib, wl, orc)
    ranks = run_cp(lib, dw, 2, paged=False)
    K, B, L = wl.top_k, wl.B, wl.L
    jobs = [4, 5]  # the last pool's jobs: its candidates are in every rank's cand
    sends_b, sends_s = [], []
    for r in ranks:
        sb = torch.zeros((len(jobs), B, K, 2), dtype=torch.int32, device="cuda")
        lib.csa2_cp_select_local_jobs(r.shard, r.kv, jobs, dw.q_idx, dw.w, r.cand, r.cand_count,
                                      K, sb, r.ws)
        ss = torch.zeros_like(sb)
        for j, x in enumerate(jobs):
            lib.csa2_cp_select_local(r.shard, r.kv, dw.q_idx[x], dw.w[x], r.cand, r.cand_count,
                                     K, ss[j], r.ws)
        torch.cuda.synchronize()
        assert torch.equal(sb, ss), int(r.shard.rank)
        sends_b.append(sb)
        sends_s.append(ss)
    gathered = torch.stack(sends_b)  # [world][J][B][K][2]
    r = ranks[0]
    idx_b = torch.full((L, B, K), -7, dtype=torch.int32, device="cuda")
    cnt_b = torch.zeros((L, B), dtype=torch.int32, device="cuda")
    lib.csa2_cp_select_merge_jobs(r.shard, gathered, jobs, B, K, idx_b, cnt_b, r.ws)
    for j, x in enumerate(jobs):
        idx_s = torch.full((B, K), -7, dtype=torch.int32, device="cuda")
        cnt_s = torch.zeros(B, dtype=torch.int32, device="cuda")
        lib.csa2_cp_select_merge(r.shard, gathered, len(jobs), j, B, K, idx_s, cnt_s, r.ws)
        torch.cuda.synchronize()
        assert torch.equal(idx_b[x], idx_s) and torch.equal(cnt_b[x], cnt_s), x
        assert torch.equal(idx_b[x], r.idx[x]) and torch.equal(cnt_b[x], r.idx_count[x]), x
    src = [0, 0, 2, 2, 4, 5]  # REUSE layers 1 and 3 read (and receive) layers 0 and 2
    for r in ranks:
        idx_a, cnt_a = r.idx.clone(), r.idx_count.clone()
        idx_a[[1, 3]] = -5  # the REUSE targets are rewritten by the calls
        loc_b = torch.full_like(r.idx_local, -9)
        lcnt_b = torch.zeros_like(r.idx_local_count)
        lib.csa2_cp_filter_layers(r.shard, src, idx_a, cnt_a, loc_b, lcnt_b, r.ws)
        idx_c, cnt_c = r.idx.clone(), r.idx_count.clone()
        idx_c[[1, 3]] = -5
        loc_s = torch.full_like(r.idx_local, -9)
        lcnt_s = torch.zeros_like(r.idx_local_count)
        for l, s_ in enumerate(src):
            reuse = s_ != l
            lib.csa2_cp_filter(r.shard, 1, idx_c[s_], cnt_c[s_], loc_s[l], lcnt_s[l], r.ws,
                               copy=idx_c[l] if reuse else None,
                               copy_count=cnt_c[l] if reuse else None)
        torch.cuda.synchronize()
        assert torch.equal(loc_b, loc_s) and torch.equal(lcnt_b, lcnt_s), int(r.shard.rank)
        assert torch.equal(idx_a, idx_c) and torch.equal(cnt_a, cnt_c)
        assert torch.equal(idx_a, r.idx) and torch.equal(cnt_a, r.idx_count)
        lib.csa2_sync_status(r.ws)
