"""GPU parity of the cache-append step (csa2_cache_append) against the oracle:
FP4 rows and window rings bit-exact, counters exact, indexer-K rows equal to
the oracle's bf16 rounding of the exact projection except where that exact
value lies within the fp32 accumulation bound of a bf16 rounding midpoint
(then either neighbour is correct).  Then a decode step on the appended
cache against the oracle's decode step on its own appended copy."""
import numpy as np
import pytest
import torch

from fp4_kv_cache_quantize_b200 import synth
from gpu_helpers import ATTN_RTOL, check_selection, rel_l2

pytestmark = pytest.mark.gpu

# fp32 accumulation of 512 products in at most 48 dependent roundings
# (16-term fused chains, then a 32-term sum): |error| <= 48 u sum|x w|, u = 2^-24.
PROJ_ERR = 64 * 2.0 ** -24


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp4_kv_cache_quantize_b200 import csa2
    return csa2


def bf16_bits(a):
    return synth.to_bf16_bits(np.asarray(a, np.float32))


def bfv(bits):
    return synth.bf16_bits_to_f32(np.asarray(bits, np.uint16)).astype(np.float64)


def dev(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda()


def check_projection(got, want, x, w):
    """got/want bf16 bits [n][64] for entries x bf16 bits [n][512]."""
    xv, wv = bfv(x), bfv(w)
    exact = xv @ wv
    bound = PROJ_ERR * (np.abs(xv) @ np.abs(wv))
    diff = got != want
    for i, j in zip(*np.nonzero(diff)):
        g, e = int(got[i, j]), int(want[i, j])
        assert abs(g - e) == 1 and (g ^ e) & 0x8000 == 0, (i, j, hex(g), hex(e))
        mid = 0.5 * (bfv([g])[0] + bfv([e])[0])
        assert abs(exact[i, j] - mid) <= bound[i, j], (i, j)


class Cache:
    """The same cache on the device and in host arrays for the oracle."""

    def __init__(self, lib, orc, B, rows, seq_stride=0, page_table=None, n_rows=None, L=0,
                 swa_pos=None, seed=0):
        rng = np.random.default_rng(seed)
        self.codes = rng.integers(0, 256, (rows, 256), dtype=np.uint8)
        self.scales = rng.integers(0, 0x70, (rows, 32), dtype=np.uint8)
        self.idxk = bf16_bits(rng.standard_normal((rows, 64)))
        self.n_rows = np.asarray(n_rows, np.int64)
        self.pt = page_table
        self.seq_stride = seq_stride
        self.L = L
        self.swa = rng.integers(0, 0x7E, (L, B, 128, 512), dtype=np.uint8) if L else None
        self.swa_pos = np.asarray(swa_pos, np.int64) if L else None
        self.swa_len = np.minimum(self.swa_pos, 128).astype(np.int32) if L else None
        self.d_codes, self.d_scales, self.d_idxk = dev(self.codes), dev(self.scales), dev(self.idxk)
        self.d_n = dev(self.n_rows.astype(np.int32))
        max_rows = int(max(self.n_rows.max(), 1))
        self.kv = lib.KVCache(self.d_codes, self.d_scales, self.d_idxk, self.d_n,
                              max_rows=max_rows, seq_stride=seq_stride,
                              page_table=None if page_table is None else dev(page_table))
        if L:
            self.d_swa = dev(self.swa)
            self.d_pos = dev(self.swa_pos.astype(np.int32))
            self.d_len = dev(self.swa_len)
        self.okv = orc.KV(self.codes.copy(), self.scales.copy(), self.idxk.copy(),
                          seq_stride=seq_stride, page_table=page_table)

    def append(self, lib, orc, x, w, xs=None):
        ws = lib.workspace(lib.WS_HEADER)
        if self.L:
            lib.csa2_cache_append(self.kv, dev(x), dev(w), ws, dev(xs), self.d_swa, self.d_pos,
                                  self.d_len)
        else:
            lib.csa2_cache_append(self.kv, dev(x), dev(w), ws)
        rc = orc.cache_append(self.okv, orc.dims(), self.n_rows, x, w, xs, self.swa,
                              self.swa_pos, self.swa_len)
        return ws, rc

    def compare(self, x_steps, w):
        assert np.array_equal(self.d_n.cpu().numpy(), self.n_rows)
        assert np.array_equal(self.d_codes.cpu().numpy(), self.okv.codes)
        assert np.array_equal(self.d_scales.cpu().numpy(), self.okv.scales)
        got = self.d_idxk.cpu().numpy().view(np.uint16)
        rows = np.nonzero((got != self.okv.idxk).any(axis=1))[0]
        if len(rows):
            # rows that differ must be appended rows within the rounding rule
            xs = {}
            for xr, rr in x_steps:
                for r, xx in zip(rr, xr):
                    xs[r] = xx
            assert set(rows.tolist()) <= set(xs), rows
            check_projection(got[rows], self.okv.idxk[rows], np.stack([xs[r] for r in rows]), w)
        if self.L:
            assert np.array_equal(self.d_swa.cpu().numpy(), self.swa)
            assert np.array_equal(self.d_pos.cpu().numpy(), self.swa_pos)
            assert np.array_equal(self.d_len.cpu().numpy(), self.swa_len)


@pytest.mark.parametrize("paged", [False, True])
def test_append_parity_over_several_steps(lib, orc, paged):
    rng = np.random.default_rng(11 + paged)
    B, L = 3, 6
    if paged:
        pt = np.array([[4, 0, -1, -1], [2, 5, 1, -1], [3, 6, 7, 8]], np.int32)
        c = Cache(lib, orc, B, 9 * 64, page_table=pt, n_rows=[62, 128, 200], L=L,
                  swa_pos=[0, 126, 1000], seed=1)
    else:
        c = Cache(lib, orc, B, 3 * 256, seq_stride=256, n_rows=[0, 100, 253], L=L,
                  swa_pos=[0, 127, 300], seed=2)
    w = bf16_bits(rng.standard_normal((512, 64)) / np.sqrt(512))
    steps = []
    for step in range(4):
        x = bf16_bits(rng.standard_normal((B, 512)) * (1.0 if step < 3 else 300.0))
        xs = bf16_bits(rng.standard_normal((L, B, 512)) * 40.0)   # some saturate at 448
        rows = [c.okv.row_of(b, int(c.n_rows[b])) for b in range(B)]
        ws, rc = c.append(lib, orc, x, w, xs)
        steps.append((x[[b for b in range(B) if rows[b] >= 0]], [r for r in rows if r >= 0]))
        if rc == 0:
            lib.csa2_sync_status(ws)
        else:   # the oracle skipped a sequence: the device must report it too
            with pytest.raises(lib.Csa2Error) as e:
                lib.csa2_sync_status(ws)
            assert e.value.status == 7
    c.compare(steps, w)


def test_append_without_window_layers(lib, orc):
    rng = np.random.default_rng(5)
    c = Cache(lib, orc, 2, 2 * 128, seq_stride=128, n_rows=[5, 127], seed=3)
    w = bf16_bits(rng.standard_normal((512, 64)) / np.sqrt(512))
    x = bf16_bits(rng.standard_normal((2, 512)))
    rows = [c.okv.row_of(b, int(c.n_rows[b])) for b in range(2)]
    ws, rc = c.append(lib, orc, x, w)
    assert rc == 0
    lib.csa2_sync_status(ws)
    c.compare([(x, rows)], w)
    ws, rc = c.append(lib, orc, x, w)       # sequence 1 is now full: skipped on both sides
    assert rc == 1 and c.n_rows.tolist() == [7, 128]
    with pytest.raises(lib.Csa2Error) as e:
        lib.csa2_sync_status(ws)
    assert e.value.status == 7
    c.compare([(x, rows), (x[:1], [c.okv.row_of(0, 6)])], w)


def test_append_host_side_errors(lib, orc):
    c = Cache(lib, orc, 1, 64, seq_stride=64, n_rows=[0], seed=4)
    ws = lib.workspace(lib.WS_HEADER)
    x = torch.zeros((1, 512), dtype=torch.int16, device="cuda")
    w = torch.zeros((512, 64), dtype=torch.int16, device="cuda")
    xs = torch.zeros((2, 1, 512), dtype=torch.int16, device="cuda")
    swa = torch.zeros((2, 1, 128, 512), dtype=torch.uint8, device="cuda")
    with pytest.raises(lib.Csa2Error) as e:
        lib.csa2_cache_append(c.kv, x, w, ws, xs, swa, None, None)
    assert e.value.status == 1
    with pytest.raises(lib.Csa2Error) as e:
        lib.csa2_cache_append(c.kv, x, w, ws[:16])
    assert e.value.status == 4
    odd = torch.zeros(513, dtype=torch.int16, device="cuda")[1:].view(1, 512)  # 2-byte offset
    with pytest.raises(lib.Csa2Error) as e:
        lib.csa2_cache_append(c.kv, odd, w, ws)
    assert e.value.status == 3


def test_decode_after_append_matches_the_oracle(lib, orc):
    """Append 3 tokens to a 3000-entry cache, then one layer group step
    (Full, Reuse) reads them: selections and attention against the oracle's
    step on its own appended cache."""
    rng = np.random.default_rng(9)
    B, L, n0 = 2, 2, [3000, 1500]
    wl = synth.make("app", seed=77, B=B, n_rows=[n + 3 for n in n0], modes=[0, 2],
                    pool_blocks=2048)
    x_all, k_all = wl.all_rows()
    w = bf16_bits(rng.standard_normal((512, 64)) / np.sqrt(512))
    codes, scales = orc.quantize_fp4(x_all)
    c = Cache(lib, orc, B, wl.pool_rows, seq_stride=wl.seq_stride, n_rows=n0, L=L,
              swa_pos=[5, 200], seed=6)
    c.codes[:], c.scales[:], c.idxk[:] = codes, scales, k_all
    for a, d_a in ((codes, c.d_codes), (scales, c.d_scales), (k_all, c.d_idxk)):
        d_a.copy_(dev(a))
    c.okv = orc.KV(codes.copy(), scales.copy(), k_all.copy(), seq_stride=wl.seq_stride)
    for step in range(3):
        x = np.stack([x_all[b * wl.seq_stride + n0[b] + step] for b in range(B)])
        xs = bf16_bits(rng.standard_normal((L, B, 512)))
        ws, rc = c.append(lib, orc, x, w, xs)
        assert rc == 0
        lib.csa2_sync_status(ws)
    # the decode step reads the device cache and the device window rings
    kv = lib.KVCache(c.d_codes, c.d_scales, c.d_idxk, c.d_n, max_rows=max(n0) + 3,
                     seq_stride=wl.seq_stride)
    grp = lib.LayerGroup(kv, wl.modes, dev(wl.q_idx), dev(wl.w_h), dev(wl.q), c.d_swa, c.d_len,
                         top_k=512, pool_blocks=2048)
    gws = lib.workspace(grp.workspace_size())
    lib.csa2_layer_group(grp, gws)
    lib.csa2_sync_status(gws)
    okv = c.okv          # the oracle's own appended cache
    dm = orc.dims()
    ref = orc.layer_group(okv, dm, c.n_rows, wl.modes, wl.q_idx, wl.w_h, wl.q, c.swa,
                          c.swa_len, top_k=512, pool_blocks=2048)
    idx, cnt = grp.idx.cpu().numpy(), grp.idx_count.cpu().numpy()
    out = grp.out.float().cpu().numpy()
    for b in range(B):
        C = int(c.n_rows[b])
        s = orc.scores(okv, dm, b, C, wl.q_idx[0, b], wl.w_h[0, b])
        check_selection(idx[0, b], int(cnt[0, b]), ref["idx"][0, b, :ref["idx_count"][0, b]],
                        lambda p: s[p], 512, cand_positions=np.arange(C), what=f"b={b}")
        for layer in range(L):
            assert rel_l2(out[layer, b], ref["out"][layer, b]) < ATTN_RTOL, (layer, b)
