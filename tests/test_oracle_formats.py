"""Pins of the oracle's FP4/FP8/bf16 formats and of its FP4 quantiser.

Every check compares the oracle with something other than itself: CUDA's host
conversion routines (tests/fmt_ref.cpp, called as a black box), torch's
float8_e4m3fn cast, the hand-worked cases of tests/golden/fp4_quant_cases.txt,
round trips of representable values, and the quantiser's error bound.
"""
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(vals):
    t = torch.tensor(np.asarray(vals, dtype=np.float32)).to(torch.bfloat16)
    back = t.float().numpy()
    assert np.array_equal(back, np.asarray(vals, dtype=np.float32)), "value not exact in bf16"
    return t.view(torch.int16).numpy().view(np.uint16)


def all_finite_bf16():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = (bits.astype(np.uint32) << 16).view(np.float32)
    return bits[np.isfinite(f)], f[np.isfinite(f)]


# ---------------------------------------------------------------- decoders
def test_e2m1_decode_matches_cuda_host_routine(orc, fmt_ref):
    for c in range(16):
        assert orc.e2m1_value(c) == fmt_ref.ref_e2m1_value(c), c


def test_e2m1_positive_grid_is_the_nvfp4_grid(orc):
    # OCP Microscaling spec E2M1 magnitudes
    assert [orc.e2m1_value(c) for c in range(8)] == [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def test_e4m3_decode_matches_torch_and_cuda(orc, fmt_ref):
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    for c in range(256):
        v = orc.e4m3_value(c)
        if np.isnan(ref[c]):
            assert np.isnan(v), c
        else:
            assert v == ref[c] == fmt_ref.ref_e4m3_value(c), c
    assert orc.e4m3_value(0x7E) == 448.0 and orc.e4m3_value(0x01) == 2.0 ** -9


def test_bf16_value_matches_torch(orc):
    bits, f = all_finite_bf16()
    sample = np.random.default_rng(0).choice(len(bits), 4000, replace=False)
    for i in sample:
        assert orc.bf16_value(int(bits[i])) == float(f[i])


def test_bf16_round_matches_torch_rne(orc):
    g = np.random.default_rng(1)
    v = np.concatenate([g.standard_normal(3000) * 10.0 ** g.integers(-6, 6, 3000),
                        # exact bf16 midpoints: ties to even
                        (bf16_mid := (np.arange(1, 200, dtype=np.float64) + 0.5) / 128.0)])
    want = torch.tensor(v, dtype=torch.float64).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = orc.bf16_round_array(v)
    assert np.array_equal(got, want)
    assert len(bf16_mid)


# ---------------------------------------------------------------- encoders
def _sweep_floats():
    g = np.random.default_rng(2)
    _, f = all_finite_bf16()
    mids = (f[:-1].astype(np.float64) + f[1:].astype(np.float64)) / 2
    rnd = (g.standard_normal(20000) * np.exp(g.uniform(-12, 8, 20000))).astype(np.float32)
    return np.concatenate([f, mids.astype(np.float32), rnd, [0.0, -0.0]]).astype(np.float32)


def test_e4m3_encode_matches_cuda_satfinite(orc, fmt_ref):
    xs = _sweep_floats()
    xs = xs[np.abs(xs) < 1e4]
    for x in xs[:: max(1, len(xs) // 40000)]:
        assert orc.e4m3_encode(float(x)) == fmt_ref.ref_e4m3_satfinite(float(x)), float(x)


def test_e4m3_encode_boundaries(orc):
    assert orc.e4m3_encode(2.0 ** -10) == 0x00            # tie to even (0)
    assert orc.e4m3_encode(np.nextafter(np.float32(2 ** -10), np.float32(1))) == 0x01
    assert orc.e4m3_encode(3 * 2.0 ** -10) == 0x02        # tie between 1 and 2 -> even 2
    assert orc.e4m3_encode(464.0) == 0x7E and orc.e4m3_encode(1e30) == 0x7E
    assert orc.e4m3_encode(-1e30) == 0xFE


def test_e2m1_encode_matches_cuda_rn(orc, fmt_ref):
    xs = _sweep_floats()
    for x in xs[:: max(1, len(xs) // 40000)]:
        assert orc.e2m1_encode(float(x)) == fmt_ref.ref_e2m1_rn(float(x)), float(x)


def test_encoders_round_trip_every_finite_code(orc):
    for c in range(256):
        v = orc.e4m3_value(c)
        if not np.isnan(v):
            assert orc.e4m3_encode(v) == c
    for c in range(16):
        assert orc.e2m1_encode(orc.e2m1_value(c) if c != 8 else -0.0) == c


# ---------------------------------------------------------------- quantiser
def _golden_cases():
    cases, cur = [], {}
    with open(os.path.join(GOLDEN, "fp4_quant_cases.txt")) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            if key == "x":
                cur = {"x": [float(v) for v in vals]}
            elif key == "scale":
                cur["scale"] = int(vals[0], 16)
            elif key == "codes":
                cur["codes"] = [int(v, 16) for v in vals]
                cases.append(cur)
    return cases


def test_quantise_golden_cases(orc):
    cases = _golden_cases()
    assert len(cases) == 8
    for i, case in enumerate(cases):
        x = bf16_bits(case["x"])
        if case["x"][1] == 0 and str(case["x"][1]).startswith("-"):
            pass
        # -0 must stay -0 in bf16
        x = np.where(np.signbit(np.asarray(case["x"], dtype=np.float32)), x | 0x8000, x).astype(np.uint16)
        codes, scales = orc.quantize_fp4(x.reshape(1, 16))
        assert scales[0, 0] == case["scale"], (i, hex(scales[0, 0]))
        assert list(codes[0]) == case["codes"], (i, [hex(c) for c in codes[0]])


def test_quantise_round_trip_of_representable_rows(orc):
    """Rows built from E2M1 grid values times an E4M3 scale, with an element
    at 6*s, come back exactly (scale recovered, codes exact)."""
    g = np.random.default_rng(3)
    grid = np.array([orc.e2m1_value(c) for c in range(16)])
    scales_ok = [c for c in range(1, 0x7F) if orc.e4m3_value(c) * 6 <= 3e38]
    rows = []
    for sc in scales_ok:
        s = orc.e4m3_value(sc)
        vals = grid[g.integers(0, 16, 16)] * s
        vals[g.integers(0, 16)] = 6 * s * (1 if g.random() < .5 else -1)
        rows.append(vals)
    x = torch.tensor(np.array(rows, dtype=np.float32)).to(torch.bfloat16)
    assert np.array_equal(x.float().numpy(), np.array(rows, dtype=np.float32))
    xb = x.view(torch.int16).numpy().view(np.uint16)
    codes, scales = orc.quantize_fp4(xb)
    assert list(scales[:, 0]) == scales_ok
    y = orc.dequantize_fp4(codes, scales)
    assert np.array_equal(y, np.array(rows, dtype=np.float64))


def test_quantise_error_bound_and_outliers(orc):
    """|x - deq| <= s for every element (half the widest grid gap, or the
    saturation loss when s rounds down); s == 0 only when amax <= 6*2^-10."""
    g = np.random.default_rng(4)
    x = g.standard_normal((64, 512)).astype(np.float32)
    x[g.random(x.shape) < 0.01] *= 50
    x[5] *= 1e-4
    xb = torch.tensor(x).to(torch.bfloat16)
    xf = xb.float().numpy().astype(np.float64)
    codes, scales = orc.quantize_fp4(xb.view(torch.int16).numpy().view(np.uint16))
    y = orc.dequantize_fp4(codes, scales)
    s = np.array([[orc.e4m3_value(int(v)) for v in row] for row in scales]).repeat(16, axis=1)
    zero = s == 0
    assert np.all(np.abs(xf - y)[~zero] <= s[~zero])
    assert np.all(np.abs(xf[zero]) <= 6 * 2.0 ** -10)
    assert np.all(y[zero] == 0)


def test_quantise_exhaustive_bf16_against_cuda_encoder(orc, fmt_ref):
    """Every finite bf16 x with |x| <= 6s, placed in a group whose amax is 6s
    (so t = s exactly), gets the code CUDA's E2M1 encoder gives x/s."""
    bits, f = all_finite_bf16()
    for sc in (0x38, 0x23, 0x01, 0x55, 0x7E):
        s = orc.e4m3_value(sc)
        anchor = bf16_bits([6 * s])[0]
        sel = np.abs(f) <= 6 * s
        xs, fs = bits[sel], f[sel]
        n = len(xs)
        pad = (-n) % 15
        xs_p = np.concatenate([xs, np.zeros(pad, np.uint16)])
        fs_p = np.concatenate([fs, np.zeros(pad, np.float32)])
        groups = xs_p.reshape(-1, 15)
        rows = np.concatenate([groups, np.full((len(groups), 1), anchor, np.uint16)], axis=1)
        codes, scales = orc.quantize_fp4(rows)
        assert np.all(scales == sc)
        lo, hi = codes & 0xF, codes >> 4
        allc = np.stack([lo, hi], axis=-1).reshape(len(groups), 16)[:, :15].ravel()
        for v, c in zip(fs_p[:n][:: max(1, n // 3000)], allc[:n][:: max(1, n // 3000)]):
            assert c == fmt_ref.ref_e2m1_rn(float(np.float32(v) / np.float32(s))), (sc, v)
