"""The exchanges of the context-parallel decode (fp4_kv_cache_quantize_b200.cp)
over torch.distributed: with world_size 2 over gloo on the CPU, DistComm's
all-gather of each exchange's buffer (block maxima, Top-k exports, attention
partials) must give every rank the rank-major stack that LocalComm builds
when both shards run in one process, the layout the merge entry points read.
Also the host-side shard arithmetic."""
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
B, NB, J, K, L = 3, 16, 2, 8, 2


def _buffers(rank):
    g = torch.Generator().manual_seed(1000 + rank)
    bm = torch.randn((B, NB), generator=g)
    sel = torch.randint(0, 1 << 30, (J, B, K, 2), generator=g, dtype=torch.int32)
    part = torch.randn(L * B * 16 * (512 + 2), generator=g)
    return bm, sel, part


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    from fp4_kv_cache_quantize_b200 import cp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        comm = cp.DistComm()
        local = cp.LocalComm(world)
        mine = _buffers(rank)
        every = [_buffers(r) for r in range(world)]
        ok = []
        for i in range(3):
            (got,) = comm.all_gather([mine[i]])
            want = local.all_gather([every[r][i] for r in range(world)])[rank]
            ok.append(bool(torch.equal(got, want)) and tuple(got.shape) ==
                      (world,) + tuple(mine[i].shape))
        dist.barrier()
        q.put((rank, ok))
    finally:
        dist.destroy_process_group()


def test_two_rank_exchanges_match_the_single_process_layout():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29700 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok in out:
        assert ok == [True, True, True], (rank, ok)


def test_shard_rows_cover_the_context():
    from fp4_kv_cache_quantize_b200 import cp
    for n in (1, 127, 128, 129, 20000, 1 << 20):
        for world in (1, 2, 3, 4, 8, 16):
            S = cp.shard_rows_for(n, world)
            assert S % 128 == 0 and S * world >= n
            assert (S - 128) * world < n  # the smallest such size


def test_local_comm_rejects_a_missing_shard():
    from fp4_kv_cache_quantize_b200 import cp
    with pytest.raises(ValueError):
        cp.LocalComm(3).all_gather([torch.zeros(2), torch.zeros(2)])


def test_local_view_checks_the_layout():
    from fp4_kv_cache_quantize_b200 import cp
    codes = torch.zeros((1024, 256), dtype=torch.uint8)
    scales = torch.zeros((1024, 32), dtype=torch.uint8)
    k = torch.zeros((1024, 64), dtype=torch.int16)
    with pytest.raises(ValueError, match="seq_stride"):
        cp.local_view(codes, scales, k, rank=0, world=4, shard_rows=256, batch=2, seq_stride=512)
    with pytest.raises(ValueError, match="64-row page"):
        cp.local_view(codes, scales, k, rank=0, world=2, shard_rows=96, batch=1,
                      page_table=torch.zeros((1, 4), dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA device"):   # the binding takes device tensors only
        cp.local_view(codes, scales, k, rank=1, world=2, shard_rows=256, batch=2, seq_stride=512)
