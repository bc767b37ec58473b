"""GPU parity of the FP4 pack / unpack kernels against the CPU oracle.

Codes and scales must match bit for bit; the dequantised bf16 values must
equal the oracle's exact products.  Calls go through the C ABI (ctypes)."""
import os

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


def gpu_quant(lib, x_bits: np.ndarray):
    x = torch.from_numpy(x_bits.view(np.int16)).cuda()
    rows, ch = x_bits.shape
    codes = torch.empty((rows, ch // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((rows, ch // 16), dtype=torch.uint8, device="cuda")
    lib.csa2_quantize_fp4(x.view(torch.bfloat16), codes, scales)
    return codes, scales


def gpu_dequant(lib, codes, scales):
    rows = codes.shape[0]
    y = torch.empty((rows, codes.shape[1] * 2), dtype=torch.bfloat16, device="cuda")
    lib.csa2_dequantize_fp4(codes, scales, y)
    return y


def f32_of(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def check_bits(lib, orc, x_bits):
    codes, scales = gpu_quant(lib, x_bits)
    oc, os_ = orc.quantize_fp4(x_bits)
    gc, gs = codes.cpu().numpy(), scales.cpu().numpy()
    bad = np.nonzero((gc != oc).any(axis=1) | (gs != os_).any(axis=1))[0]
    assert len(bad) == 0, f"{len(bad)} rows differ, first {bad[:5]}"
    y = gpu_dequant(lib, codes, scales).view(torch.int16).cpu().numpy().view(np.uint16)
    want = orc.dequantize_fp4(oc, os_)
    assert np.array_equal(f32_of(y).astype(np.float64), want)


def test_quant_random_rows_with_outliers_and_tiny_groups(lib, orc):
    g = np.random.default_rng(0)
    x = g.standard_normal((777, 512)).astype(np.float32)
    x[g.random(x.shape) < 0.001] *= 50
    x[3] *= 1e-3            # tiny groups -> zero and subnormal scales
    x[4] *= 1e-5
    x[5] = 0.0
    x[6, ::2] = -0.0
    x[7] *= 1e4             # saturating scale
    check_bits(lib, orc, synth.to_bf16_bits(x))


def test_quant_exhaustive_bf16_patterns(lib, orc):
    """Every finite bf16 pattern, in groups whose amax pins the scale."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = f32_of(bits)
    bits = bits[np.isfinite(f)]
    rows = []
    for anchor in (6.0, 6.0 * 0.171875, 6 * 2.0 ** -9, 6 * 448.0, 1e30):
        a = synth.to_bf16_bits(np.array([anchor], np.float32))[0]
        grp = np.concatenate([bits, np.zeros((-len(bits)) % 15, np.uint16)]).reshape(-1, 15)
        rows.append(np.concatenate([grp, np.full((len(grp), 1), a, np.uint16)], axis=1))
    grp = np.concatenate(rows)
    grp = np.concatenate([grp, np.zeros(((-len(grp)) % 32, 16), np.uint16)])
    check_bits(lib, orc, np.ascontiguousarray(grp.reshape(-1, 512)))


@pytest.mark.parametrize("rows,ch", [(1, 16), (3, 48), (5, 512), (129, 512)])
def test_quant_ragged_shapes(lib, orc, rows, ch):
    g = np.random.default_rng(rows * ch)
    check_bits(lib, orc, synth.to_bf16_bits(g.standard_normal((rows, ch)).astype(np.float32)))


def test_quant_zero_rows_and_bad_shape(lib):
    x = torch.zeros((0, 512), dtype=torch.bfloat16, device="cuda")
    codes = torch.zeros((0, 256), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((0, 32), dtype=torch.uint8, device="cuda")
    lib.csa2_quantize_fp4(x, codes, scales)
    with pytest.raises(lib.Csa2Error) as e:
        lib.csa2_quantize_fp4(torch.zeros((2, 24), dtype=torch.bfloat16, device="cuda"),
                              torch.zeros((2, 12), dtype=torch.uint8, device="cuda"),
                              torch.zeros((2, 2), dtype=torch.uint8, device="cuda"))
    assert e.value.status == 2


@pytest.mark.slow
def test_quant_full_size_1M_rows_every_row(lib, orc):
    """The 1,048,576 x 512 workload with 0.1% x50 outliers, quantised on the
    GPU in one launch (the launch the microbenchmark times): every row's
    codes and scales bit-exact against the oracle (chunks of 4,096 rows on
    host threads), and the whole output's dequant round trip checked by
    property."""
    wl = synth.config(1)
    rows = wl.pool_rows
    x = torch.empty((rows, 512), dtype=torch.int16, device="cuda")
    for c in range(wl.n_chunks):
        xc = wl.x_chunk(c)
        r0 = c * synth.CHUNK_ROWS
        x[r0:r0 + len(xc)] = torch.from_numpy(xc.view(np.int16)).cuda()
    codes = torch.empty((rows, 256), dtype=torch.uint8, device="cuda")
    scales = torch.empty((rows, 32), dtype=torch.uint8, device="cuda")
    lib.csa2_quantize_fp4(x.view(torch.bfloat16), codes, scales)
    codes_h, scales_h = codes.cpu().numpy(), scales.cpu().numpy()

    def chunk_matches(c):
        xc = wl.x_chunk(c)
        r0 = c * synth.CHUNK_ROWS
        oc, os_ = orc.quantize_fp4(xc)   # the oracle runs without the GIL (ctypes)
        return (np.array_equal(codes_h[r0:r0 + len(xc)], oc) and
                np.array_equal(scales_h[r0:r0 + len(xc)], os_))

    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max(1, min(32, os.cpu_count() or 1))) as ex:
        ok = list(ex.map(chunk_matches, range(wl.n_chunks)))
    bad = [c for c, v in enumerate(ok) if not v]
    assert not bad, f"chunks of {synth.CHUNK_ROWS} rows that differ from the oracle: {bad[:10]}"
    # property over every row: |x - deq| <= scale, elementwise
    y = gpu_dequant(lib, codes, scales).float()
    xf = x.view(torch.bfloat16).float()
    s = scales.view(torch.float8_e4m3fn).float().repeat_interleave(16, dim=1)
    assert bool(((xf - y).abs() <= s + (s == 0) * 6 * 2.0 ** -10).all())
