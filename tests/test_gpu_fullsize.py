"""Full-size parity of the decode step on the benchmark workloads, in the
launch configuration bench.py times: the HSI group (8 x 131,072), the
1M-context 20-layer decoder stack, and the ragged paged batch (64 sequences,
16K..131K entries).  The GPU quantises its cache with its own pack kernel
(bit-exact against the oracle in test_gpu_quant); the oracle quantises, with
its own encoder, only the rows that the selections make it read, found by a
first oracle pass (selection never reads main-KV codes).  Every layer's
indices, the pool and every attention output are compared."""
import numpy as np
import pytest
import torch

from fp4_kv_cache_quantize_b200 import synth
from gpu_helpers import DeviceWorkload
from test_gpu_group import compare_group, run_group

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp4_kv_cache_quantize_b200 import csa2
    return csa2


def oracle_two_pass(orc, wl, idxk_np):
    dm = orc.dims()
    codes = np.zeros((wl.pool_rows, 256), np.uint8)
    scales = np.zeros((wl.pool_rows, 32), np.uint8)
    kv = orc.KV(codes, scales, idxk_np, seq_stride=wl.seq_stride, page_table=wl.page_table)
    args = (kv, dm, wl.n_rows, wl.modes, wl.q_idx, wl.w_h, wl.q, wl.swa, wl.swa_len)
    kw = dict(top_k=wl.top_k, pool_blocks=wl.pool_blocks, sm_scale=float(np.float32(512 ** -0.5)))
    first = orc.layer_group(*args, **kw)
    rows = set()
    for l in range(wl.L):
        for b in range(wl.B):
            rows.update(wl.row_of(b, first["idx"][l, b, :first["idx_count"][l, b]]).tolist())
    rows = np.array(sorted(rows), dtype=np.int64)
    xs, _ = wl.rows(rows)
    c, s = orc.quantize_fp4(xs)
    kv.codes[rows] = c
    kv.scales[rows] = s
    return kv, orc.layer_group(*args, **kw)


@pytest.mark.parametrize("k", [2, 3, 4])
def test_full_size_parity(lib, orc, k):
    wl = synth.config(k)
    dw = DeviceWorkload(lib, wl, orc, oracle_codes=False)
    grp = run_group(lib, dw)
    kv, ref = oracle_two_pass(orc, wl, dw.idxk_np)
    compare_group(orc, dw, grp, kv=kv, ref=ref)
