"""The context-parallel driver (fp4_kv_cache_quantize_b200.cp.cp_layer_group)
on the CPU: its csa2_cp_* calls are replaced by CPU stand-ins written from the
definitions in include/csa2.h on top of the oracle, so that the driver's order
of calls, its three exchanges, its job batching, its REUSE copies and its
window placement run as two gloo ranks (DistComm) and as 1 and 3 shards in one
process (LocalComm).  The stand-ins rank by fp32 keys like the library; every
run must give the same indices and pool, those must match the oracle's
one-device layer group within the selection tolerance, and the merged output
its output within the attention tolerance."""
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FULL, REINDEX, REUSE = 0, 1, 2
MODES = [FULL, REUSE, REINDEX, REUSE, FULL, REINDEX]
TOP_K, POOL, SEED = 64, 128, 77
N_ROWS = [3000, 700]
SM = float(np.float32(512 ** -0.5))
LOG2E = 1.4426950408889634


def _workload():
    from fp4_kv_cache_quantize_b200 import synth
    return synth.make("cp_driver", seed=SEED, B=len(N_ROWS), n_rows=N_ROWS, modes=MODES,
                      top_k=TOP_K, pool_blocks=POOL, swa_len=[128, 40])


def _key(f32: np.ndarray) -> np.ndarray:
    """The library's order-preserving key of fp32 values (0 = none)."""
    u = np.asarray(f32, np.float32).view(np.uint32)
    return np.where(u & 0x80000000, ~u, u | 0x80000000).astype(np.uint32)


class ShardKV:
    """A shard's rows as an oracle cache, plus what CPRank reads."""

    def __init__(self, orc, codes, scales, k, S, B):
        self.okv = orc.KV(codes, scales, k, seq_stride=S)
        self.codes, self.scales = codes, scales
        self.batch = B
        self.n_rows = torch.zeros(B, dtype=torch.int32)


class FakeLib:
    """CPU stand-ins of the csa2_cp_* entry points (layouts as in csa2.h)."""
    FULL, REINDEX, REUSE, BLK, H, D = FULL, REINDEX, REUSE, 8, 16, 512

    def __init__(self, orc, wl):
        from fp4_kv_cache_quantize_b200 import csa2
        self.orc, self.wl, self.dm = orc, wl, orc.dims()
        self.CpShard, self.Csa2Error = csa2.CpShard, csa2.Csa2Error
        self.e4m3 = np.array([orc.e4m3_value(i) for i in range(256)], np.float64)

    @staticmethod
    def workspace(n, device=None):
        return torch.zeros(max(int(n), 256), dtype=torch.uint8)

    @staticmethod
    def csa2_cp_workspace_size(shard, B, L, K):
        return 256

    @staticmethod
    def csa2_cp_partial_floats(B, L):
        return L * B * 16 * 514

    def csa2_cp_local_rows(self, sh, n_rows, local, ws):
        lo = sh.rank * sh.shard_rows
        local.copy_((n_rows.long() - lo).clamp(0, sh.shard_rows).int())

    def csa2_cp_block_max(self, sh, kv, q_idx, w, bm, ws):
        for b in range(kv.batch):
            C = int(kv.n_rows[b])
            s = self.orc.scores(kv.okv, self.dm, b, C, q_idx[b].numpy().view(np.uint16),
                                w[b].numpy())[:C]
            m = self.orc.block_max(s.astype(np.float32).astype(np.float64), 8)
            bm[b, :len(m)] = torch.from_numpy(m.astype(np.float32))

    def csa2_cp_pool(self, sh, bm_all, n_rows, P, pool, pool_count, ws):
        for b in range(pool.shape[0]):
            nblk = -(-int(n_rows[b]) // 8)
            v = bm_all[:, b].reshape(-1)[:nblk].double().numpy()
            sel = self.orc.pool(v, P) if nblk else np.zeros(0, np.int32)
            pool[b].fill_(-1)
            pool[b, :len(sel)] = torch.from_numpy(sel.astype(np.int32))
            pool_count[b] = len(sel)

    def csa2_cp_filter(self, sh, unit, lst, count, out, out_count, ws, copy=None,
                       copy_count=None):
        lo = sh.rank * (sh.shard_rows // unit)
        hi = lo + sh.shard_rows // unit
        for b in range(lst.shape[0]):
            x = lst[b, :int(count[b])]
            keep = x[(x >= lo) & (x < hi)] - lo
            m = min(len(keep), out.shape[-1])
            out[b].fill_(-1)
            out[b, :m] = keep[:m]
            out_count[b] = m
        if copy is not None:
            copy.copy_(lst)
            copy_count.copy_(count)

    def csa2_cp_select_local(self, sh, kv, q_idx, w, cand, cand_count, top_k, send, ws):
        send.zero_()
        send[..., 1] = -1
        for b in range(kv.batch):
            C = int(kv.n_rows[b])
            blocks = cand[b, :int(cand_count[b])].numpy()
            pos = np.array([8 * j + i for j in blocks for i in range(8) if 8 * j + i < C],
                           np.int64)
            if len(pos) == 0:
                continue
            s = self.orc.scores(kv.okv, self.dm, b, C, q_idx[b].numpy().view(np.uint16),
                                w[b].numpy())[:C]
            f = s[pos].astype(np.float32)
            picked = self.orc.select_topk(f.astype(np.float64), top_k, ids=pos).astype(np.int64)
            keys = _key(s[picked].astype(np.float32))
            n = len(picked)
            send[b, :n, 0] = torch.from_numpy(keys.view(np.int32))
            send[b, :n, 1] = torch.from_numpy((picked + sh.rank * sh.shard_rows).astype(np.int32))

    def csa2_cp_select_merge(self, sh, gathered, n_jobs, job, B, top_k, idx, idx_count, ws):
        g = gathered[:, job]  # [world][B][top_k][2]
        for b in range(B):
            keys = g[:, b, :, 0].reshape(-1).numpy().view(np.uint32)
            pos = g[:, b, :, 1].reshape(-1).numpy()
            ok = keys != 0
            order = np.lexsort((pos[ok], -keys[ok].astype(np.int64)))
            top = np.sort(pos[ok][order][:top_k])
            idx[b].fill_(-1)
            idx[b, :len(top)] = torch.from_numpy(top.astype(np.int32))
            idx_count[b] = len(top)

    CP_MAX_JOBS = 8

    def csa2_cp_select_local_jobs(self, sh, kv, layers, q_idx, w, cand, cand_count, top_k, send,
                                  ws):
        assert 1 <= len(layers) <= self.CP_MAX_JOBS
        for j, x in enumerate(layers):  # job j: layer x's queries, export slot j
            self.csa2_cp_select_local(sh, kv, q_idx[x], w[x], cand, cand_count, top_k, send[j],
                                      ws)

    def csa2_cp_select_merge_jobs(self, sh, gathered, layers, B, top_k, idx, idx_count, ws):
        for j, x in enumerate(layers):  # gathered job j -> layer x
            self.csa2_cp_select_merge(sh, gathered, len(layers), j, B, top_k, idx[x],
                                      idx_count[x], ws)

    def csa2_cp_filter_layers(self, sh, src, idx, idx_count, idx_local, idx_local_count, ws):
        for l, s_ in enumerate(src):
            assert s_ <= l and src[s_] == s_
            reuse = s_ != l
            self.csa2_cp_filter(sh, 1, idx[s_], idx_count[s_], idx_local[l], idx_local_count[l],
                                ws, copy=idx[l] if reuse else None,
                                copy_count=idx_count[l] if reuse else None)

    def csa2_cp_attn_partial(self, sh, kv, q, swa, swa_len, idx_local, idx_count, sm_scale,
                             partial, ws):
        L, B = q.shape[0], q.shape[1]
        O = partial[:L * B * 16 * 512].view(L, B, 16, 512)
        ML = partial[L * B * 16 * 512:].view(L, B, 16, 2)
        for l in range(L):
            for b in range(B):
                rows = idx_local[l, b, :int(idx_count[l, b])].numpy().astype(np.int64)
                r = b * sh.shard_rows + rows
                vals = [self.orc.dequantize_fp4(kv.codes[r], kv.scales[r])] if len(r) else []
                nw = int(swa_len[b])
                if nw:
                    vals.append(self.e4m3[swa[l, b, :nw].numpy()])
                if not vals:
                    O[l, b] = 0
                    ML[l, b, :, 0] = -np.inf
                    ML[l, b, :, 1] = 0
                    continue
                V = np.concatenate(vals)
                qf = q[l, b].float().double().numpy()
                logit = qf @ V.T * sm_scale
                m = logit.max(axis=1, keepdims=True)
                p = np.exp(logit - m)
                O[l, b] = torch.from_numpy(p @ V)
                ML[l, b, :, 0] = torch.from_numpy(m[:, 0] * LOG2E)
                ML[l, b, :, 1] = torch.from_numpy(p.sum(1))

    def csa2_cp_attn_combine(self, sh, gathered, L, B, out, ws):
        O = gathered[:, :L * B * 16 * 512].reshape(-1, L, B, 16, 512).double()
        ML = gathered[:, L * B * 16 * 512:].reshape(-1, L, B, 16, 2).double()
        m = ML[..., 0]
        mx = m.max(0).values
        f = torch.where(torch.isinf(m), torch.zeros_like(m), torch.exp2(m - mx))
        den = (f * ML[..., 1]).sum(0)
        num = (f[..., None] * O).sum(0)
        res = torch.where(den[..., None] > 0, num / den.clamp_min(1e-300)[..., None],
                          torch.zeros_like(num))
        out.copy_(res.to(torch.bfloat16))


def _shard_ranks(cp, orc, wl, x_codes, x_scales, k, world, ranks):
    """CPRank objects of the given shard indices over the workload's rows."""
    S = cp.shard_rows_for(max(N_ROWS), world)
    B = wl.B
    out = []
    for r in ranks:
        codes = np.zeros((B * S, 256), np.uint8)
        scales = np.zeros((B * S, 32), np.uint8)
        kk = np.zeros((B * S, 64), np.uint16)
        for b in range(B):
            lo, hi = r * S, min(int(wl.n_rows[b]), (r + 1) * S)
            if hi > lo:
                rows = wl.row_of(b, np.arange(lo, hi))
                codes[b * S:b * S + hi - lo] = x_codes[rows]
                scales[b * S:b * S + hi - lo] = x_scales[rows]
                kk[b * S:b * S + hi - lo] = k[rows]
        kv = ShardKV(orc, codes, scales, kk, S, B)
        out.append(cp.CPRank(kv, rank=r, world=world, shard_rows=S, n_layers=wl.L, top_k=TOP_K,
                             pool_blocks=POOL))
    return out


def _step(cp, wl, ranks, comm):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(  # noqa: E731
        a.view(np.int16) if a.dtype == np.uint16 else a))
    cp.cp_layer_group(ranks, comm, MODES, t(wl.n_rows.astype(np.int32)), t(wl.q_idx), t(wl.w_h),
                      t(wl.q).view(torch.bfloat16), t(wl.swa), t(wl.swa_len), sm_scale=SM)
    return [(r.idx.numpy().copy(), r.idx_count.numpy().copy(), r.pool.numpy().copy(),
             r.pool_count.numpy().copy(), r.out.float().numpy().copy()) for r in ranks]


def _setup():
    sys.path.insert(0, ROOT)
    import oracle
    oracle.build()
    from fp4_kv_cache_quantize_b200 import cp
    wl = _workload()
    x, k = wl.all_rows()
    codes, scales = oracle.quantize_fp4(x)
    cp.csa2 = FakeLib(oracle, wl)
    return oracle, cp, wl, codes, scales, k


def _worker(rank, world, port, q):
    orc, cp, wl, codes, scales, k = _setup()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ranks = _shard_ranks(cp, orc, wl, codes, scales, k, world, [rank])
        res = _step(cp, wl, ranks, cp.DistComm())
        dist.barrier()
        q.put((rank, res[0]))
    finally:
        dist.destroy_process_group()


def _same(a, b):
    for x, y in zip(a[:4], b[:4]):
        assert np.array_equal(x, y)
    assert np.allclose(a[4], b[4], rtol=0, atol=2e-2 * max(1.0, np.abs(b[4]).max()))


def test_driver_over_two_gloo_ranks_and_one_process(orc):
    import importlib
    from gpu_helpers import ATTN_RTOL, check_selection, rel_l2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29800 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    dist_res = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0

    _, cp, wl, codes, scales, k = _setup()
    try:
        one = _step(cp, wl, _shard_ranks(cp, orc, wl, codes, scales, k, 1, [0]),
                    cp.LocalComm(1))[0]
        three = _step(cp, wl, _shard_ranks(cp, orc, wl, codes, scales, k, 3, [0, 1, 2]),
                      cp.LocalComm(3))
    finally:
        from fp4_kv_cache_quantize_b200 import cp as cp_mod
        importlib.reload(cp_mod)
    for res in [dist_res[0], dist_res[1]] + three:
        _same(res, one)

    # against the oracle's one-device layer group
    kv = orc.KV(codes, scales, k, seq_stride=wl.seq_stride)
    dm = orc.dims()
    ref = orc.layer_group(kv, dm, wl.n_rows, MODES, wl.q_idx, wl.w_h, wl.q, wl.swa, wl.swa_len,
                          top_k=TOP_K, pool_blocks=POOL, sm_scale=SM)
    idx, cnt, pool, pcnt, out = one
    for b in range(wl.B):
        C = int(wl.n_rows[b])
        for l in range(wl.L):
            if MODES[l] == REUSE:
                continue
            s = orc.scores(kv, dm, b, C, wl.q_idx[l, b], wl.w_h[l, b])
            check_selection(idx[l, b], int(cnt[l, b]), ref["idx"][l, b, :ref["idx_count"][l, b]],
                            lambda p, s=s: s[p], TOP_K, what=f"layer {l} b={b}")
        for l in range(wl.L):
            assert rel_l2(out[l, b].astype(np.float64), ref["out"][l, b]) <= ATTN_RTOL, (l, b)
