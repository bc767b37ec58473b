"""Context-parallel decode of a CSA2 layer group (include/csa2.h, section
"context-parallel decode").

Every sequence's positions are cut into `world` contiguous shards of
`shard_rows` rows; shard r (positions [r*S, (r+1)*S)) lives on rank r.  Every
step of the decode runs in libcsa2's kernels through the csa2_cp_* entry
points; this module only orders the calls and performs the three exchanges
as all-gathers through a communicator:

  * DistComm -- one rank per process over torch.distributed (NCCL between
    GPUs, gloo on CPU for the host-side tests);
  * LocalComm -- every shard in one process on one device, the exchange a
    device copy: the shards' kernels run one after the other and never wait
    on each other.

Per FULL layer (and per REINDEX layer without a pool) the exchanges carry the
shard's block maxima (4 bytes per 8 rows); per selecting layer, or per FULL
layer with its pool-sharing REINDEX layers batched, the shard's Top-k as
(key, position) pairs (8 bytes each); once per step, every layer's attention
partial (16 x 514 floats per layer and sequence).
"""
from __future__ import annotations

import torch

from . import csa2

FULL, REINDEX, REUSE = csa2.FULL, csa2.REINDEX, csa2.REUSE


def shard_rows_for(max_rows: int, world: int) -> int:
    """The smallest shard size (a multiple of 128 rows) that covers max_rows."""
    per = -(-max(int(max_rows), 1) // int(world))
    return -(-per // 128) * 128


class LocalComm:
    """All shards in this process: all_gather stacks the shards' buffers in
    rank order (one device copy) and hands the result to every shard."""

    def __init__(self, world: int):
        self.world = int(world)

    def all_gather(self, sends):
        if len(sends) != self.world:
            raise ValueError(f"{len(sends)} buffers for {self.world} shards")
        g = torch.stack([s.contiguous() for s in sends])
        return [g] * self.world


class DistComm:
    """One shard per process: all_gather over a torch.distributed group."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.world = dist.get_world_size(group)
        self.nccl = dist.get_backend(group) == "nccl"

    def all_gather(self, sends):
        if len(sends) != 1:
            raise ValueError("DistComm runs one shard per process")
        send = sends[0].contiguous()
        out = send.new_empty((self.world,) + tuple(send.shape))
        if self.nccl:
            self.dist.all_gather_into_tensor(out, send, group=self.group)
        else:
            self.dist.all_gather(list(out.unbind(0)), send, group=self.group)
        return [out]


def local_view(codes, scales, idx_k, *, rank: int, world: int, shard_rows: int, batch: int,
               seq_stride: int = 0, page_table=None) -> csa2.KVCache:
    """The view of shard `rank` inside one device's cache of all positions:
    contiguous sequences need seq_stride >= world * shard_rows (the shard is
    the same row pool from row rank * shard_rows on); a paged cache gives the
    shard its columns of the page table (-1 past the table).  Its n_rows is a
    fresh device tensor that csa2_cp_local_rows fills."""
    dev = codes.device
    n_local = torch.zeros(batch, dtype=torch.int32, device=dev)
    S = int(shard_rows)
    if page_table is None:
        if seq_stride < world * S:
            raise ValueError(f"seq_stride {seq_stride} < world x shard_rows {world * S}")
        r0 = rank * S
        return csa2.KVCache(codes[r0:], scales[r0:], idx_k[r0:], n_local, max_rows=S,
                            seq_stride=seq_stride)
    if S % 64:
        raise ValueError("shard_rows must be a multiple of the 64-row page")
    pp = S // 64
    pt = torch.full((batch, pp), -1, dtype=torch.int32, device=dev)
    lo = rank * pp
    hi = min(lo + pp, page_table.shape[1])
    if hi > lo:
        pt[:, :hi - lo] = page_table[:, lo:hi]
    return csa2.KVCache(codes, scales, idx_k, n_local, max_rows=S, page_table=pt)


class CPRank:
    """One shard's state for a layer group: its view of the cache, its
    workspace, and its exchange and output buffers."""

    def __init__(self, kv: csa2.KVCache, *, rank: int, world: int, shard_rows: int,
                 n_layers: int, top_k: int = 512, pool_blocks: int = 2048):
        B = kv.batch
        dev = kv.n_rows.device
        self.kv, self.L, self.B, self.top_k, self.pool_blocks = kv, n_layers, B, top_k, pool_blocks
        self.shard = csa2.CpShard(rank, world, shard_rows)
        nbytes = csa2.csa2_cp_workspace_size(self.shard, B, n_layers, top_k)
        if nbytes == 0:
            raise csa2.Csa2Error(2, f"bad shard or sizes: rank {rank} world {world} "
                                    f"shard_rows {shard_rows}")
        self.ws = csa2.workspace(nbytes, dev)
        P = pool_blocks if pool_blocks > 0 else top_k
        i32 = dict(dtype=torch.int32, device=dev)
        self.bm = torch.empty((B, shard_rows // csa2.BLK), dtype=torch.float32, device=dev)
        self.pool = torch.full((B, P), -1, **i32)
        self.pool_count = torch.zeros(B, **i32)
        self.blocks = torch.full((B, P), -1, **i32)
        self.blocks_count = torch.zeros(B, **i32)
        self.cand = torch.empty((B, P), **i32)
        self.cand_count = torch.zeros(B, **i32)
        self.send_sel = torch.empty((n_layers, B, top_k, 2), **i32)
        self.idx = torch.empty((n_layers, B, top_k), **i32)
        self.idx_count = torch.zeros((n_layers, B), **i32)
        self.idx_local = torch.empty((n_layers, B, top_k), **i32)
        self.idx_local_count = torch.zeros((n_layers, B), **i32)
        self.partial = torch.empty(csa2.csa2_cp_partial_floats(B, n_layers), dtype=torch.float32,
                                   device=dev)
        self.out = torch.empty((n_layers, B, csa2.H, csa2.D), dtype=torch.bfloat16, device=dev)
        self.no_window = torch.zeros(B, **i32)


def cp_layer_group(ranks, comm, modes, n_rows, q_idx, w, q, swa, swa_len, *,
                   sm_scale=None, window_rank: int = 0):
    """One decode step of a layer group over context shards.

    ranks: the CPRank objects this process runs (one with DistComm, all with
    LocalComm).  n_rows int32 [B] global visible rows; q_idx bf16
    [L][B][8][64], w fp32 [L][B][8], q bf16 [L][B][16][512], swa E4M3
    [L][B][128][512], swa_len int32 [B]: the same step inputs as
    csa2_layer_group, on every rank (the window is read on window_rank only).
    Results land in each rank's idx / idx_count ([L][B][top_k], [L][B]),
    pool / pool_count (the last FULL layer's pool) and out ([L][B][16][512])."""
    modes = [int(m) for m in modes]
    L = len(modes)
    r0 = ranks[0]
    if L != r0.L or L < 1 or modes[0] != FULL:
        raise ValueError("modes must match the ranks' layer count and start with FULL")
    if sm_scale is None:
        sm_scale = csa2.D ** -0.5
    B, K, hsi = r0.B, r0.top_k, r0.pool_blocks > 0
    P = r0.pool_blocks if hsi else K

    for r in ranks:
        csa2.csa2_cp_local_rows(r.shard, n_rows, r.kv.n_rows, r.ws)

    # Indexer: one scan + pool exchange per FULL layer (and per REINDEX layer
    # without a pool), one selection exchange for it and the REINDEX layers
    # that share its pool.
    for l in range(L):
        m = modes[l]
        if m == REUSE or (m == REINDEX and hsi):
            continue
        for r in ranks:
            csa2.csa2_cp_block_max(r.shard, r.kv, q_idx[l], w[l], r.bm, r.ws)
        bm_all = comm.all_gather([r.bm for r in ranks])
        jobs = [l]
        if hsi and m == FULL:
            for x in range(l + 1, L):
                if modes[x] == FULL:
                    break
                if modes[x] == REINDEX:
                    jobs.append(x)
        for r, g in zip(ranks, bm_all):
            # the global candidate blocks (the pool, or top_k blocks without
            # one), then those this shard owns, as local block ids
            blocks, count = (r.pool, r.pool_count) if hsi else (r.blocks, r.blocks_count)
            csa2.csa2_cp_pool(r.shard, g, n_rows, P, blocks, count, r.ws)
            csa2.csa2_cp_filter(r.shard, csa2.BLK, blocks, count, r.cand, r.cand_count, r.ws)
        # the jobs' local selections (one launch pair per chunk of jobs), one
        # exchange and one merge launch per chunk
        for c0 in range(0, len(jobs), csa2.CP_MAX_JOBS):
            chunk = jobs[c0:c0 + csa2.CP_MAX_JOBS]
            J = len(chunk)
            for r in ranks:
                csa2.csa2_cp_select_local_jobs(r.shard, r.kv, chunk, q_idx, w, r.cand,
                                               r.cand_count, K, r.send_sel[:J], r.ws)
            sel_all = comm.all_gather([r.send_sel[:J] for r in ranks])
            for r, g in zip(ranks, sel_all):
                csa2.csa2_cp_select_merge_jobs(r.shard, g, chunk, B, K, r.idx, r.idx_count, r.ws)

    # Attention: each shard over the selected rows it owns (+ the window on
    # window_rank), one exchange of the partials, one merge.
    # every layer's source of indices: itself, or (REUSE) the latest FULL /
    # REINDEX layer, whose indices it also publishes
    src, cur = [], 0
    for l in range(L):
        if modes[l] != REUSE:
            cur = l
        src.append(cur)
    for r in ranks:
        csa2.csa2_cp_filter_layers(r.shard, src, r.idx, r.idx_count, r.idx_local,
                                   r.idx_local_count, r.ws)
        win = swa_len if int(r.shard.rank) == window_rank else r.no_window
        csa2.csa2_cp_attn_partial(r.shard, r.kv, q, swa, win, r.idx_local, r.idx_local_count,
                                  sm_scale, r.partial, r.ws)
    part_all = comm.all_gather([r.partial for r in ranks])
    for r, g in zip(ranks, part_all):
        csa2.csa2_cp_attn_combine(r.shard, g, L, B, r.out, r.ws)
