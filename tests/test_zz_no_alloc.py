"""csa2_index_full_noalloc: the Full-mode indexer for callers that cannot
allocate device memory (its scratch is a static device array inside the
library).  Its outputs must equal csa2_index_full's, with a caller workspace,
on two calls in a row (the second call reuses the scratch the first one
left behind).  Named to be collected last."""
import numpy as np
import pytest
import torch

from fp4_kv_cache_quantize_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp4_kv_cache_quantize_b200 import csa2
    return csa2


def _setup(lib, n_rows, seed, paged=False):
    wl = synth.make("na", seed=seed, B=len(n_rows), n_rows=n_rows, modes=[0], paged=paged)
    x, k = wl.all_rows()
    xt = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    codes = torch.empty((wl.pool_rows, 256), dtype=torch.uint8, device="cuda")
    scales = torch.empty((wl.pool_rows, 32), dtype=torch.uint8, device="cuda")
    lib.csa2_quantize_fp4(xt, codes, scales)
    idxk = torch.from_numpy(k.view(np.int16)).cuda()
    n = torch.from_numpy(wl.n_rows.astype(np.int32)).cuda()
    pt = None if wl.page_table is None else torch.from_numpy(wl.page_table).cuda()
    kv = lib.KVCache(codes, scales, idxk, n, max_rows=int(wl.n_rows.max()),
                     seq_stride=wl.seq_stride, page_table=pt)
    q_idx = torch.from_numpy(wl.q_idx[0].view(np.int16)).cuda()
    w = torch.from_numpy(wl.w_h[0]).cuda()
    return kv, q_idx, w


def _outputs(B, top_k, pool_blocks):
    return (torch.full((B, top_k), -7, dtype=torch.int32, device="cuda"),
            torch.full((B,), -7, dtype=torch.int32, device="cuda"),
            torch.full((B, pool_blocks), -7, dtype=torch.int32, device="cuda"),
            torch.full((B,), -7, dtype=torch.int32, device="cuda"))


@pytest.mark.parametrize("n_rows,paged", [([20000, 7777], False), ([9000, 130, 4099], True)])
def test_noalloc_matches_workspace_entry_point_twice(lib, n_rows, paged):
    B, top_k, pb = len(n_rows), 512, 2048
    kv, q_idx, w = _setup(lib, n_rows, seed=1234 + len(n_rows), paged=paged)
    ref = _outputs(B, top_k, pb)
    ws = lib.workspace(lib.csa2_index_workspace_size(kv, top_k, pb))
    lib.csa2_workspace_init(ws)
    lib.csa2_index_full(kv, q_idx, w, top_k, pb, *ref, ws)
    lib.csa2_sync_status(ws)
    want = [t.cpu().numpy() for t in ref]
    for call in range(2):
        got = _outputs(B, top_k, pb)
        lib.csa2_index_full_noalloc(kv, q_idx, w, top_k, pb, *got)
        torch.cuda.synchronize()
        for name, g, e in zip(("idx", "idx_count", "pool", "pool_count"), got, want):
            assert np.array_equal(g.cpu().numpy(), e), (call, name)


def test_noalloc_rejects_more_than_its_scratch(lib):
    # 8 sequences of 1M positions need 8 x 131072 x 4 bytes of block maxima
    kv, q_idx, w = _setup(lib, [64], seed=5)
    n = torch.full((8,), 64, dtype=torch.int32, device="cuda")
    big = lib.KVCache(kv.codes, kv.scales, kv.idx_k, n, max_rows=1 << 20, seq_stride=1 << 20)
    big.view.pool_rows = 8 << 20      # host-side shape only: rejected before any launch
    out = _outputs(8, 512, 2048)
    with pytest.raises(lib.Csa2Error) as e:
        lib.csa2_index_full_noalloc(big, torch.zeros((8, 8, 64), dtype=torch.int16,
                                                     device="cuda"),
                                    torch.zeros((8, 8), device="cuda"), 512, 2048, *out)
    assert e.value.status == 4
    assert "static scratch" in str(e.value)
