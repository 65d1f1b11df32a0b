"""Pins for the oracle's scalar formats: decoders, RNE encoders, bf16 rounding.

Each check ties the oracle to something other than itself: the element and
scale types named on the pages (e2m1 codes, float8_e4m3fn scales, and
float8_e8m0fnu MX scales; hao-ai-lab-FastVideo nvfp4_config.py module
docstring, vllm-omni mxfp8_config.py DiffusionMXFP8Config docstring) as torch
implements them, closed forms, and hand-worked points in tests/golden/.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from tests._golden import e2m1_points

# The eight e2m1 magnitudes, listed (not computed) for codes 0..7.
E2M1_LISTED = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_decode_matches_listed_table():
    for code in range(16):
        v = oracle.e2m1_value(code)
        ref = E2M1_LISTED[code & 7]
        assert v == (-ref if code & 8 else ref)
        assert math.copysign(1.0, v) == (-1.0 if code & 8 else 1.0)


def test_e4m3_decode_matches_torch_float8_e4m3fn():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = np.array([oracle.e4m3_value(b) for b in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours))
    assert nan.sum() == 2  # 0x7f and 0xff
    assert np.array_equal(ref[~nan], ours[~nan])
    assert oracle.e4m3_value(0x7E) == 448.0 and oracle.e4m3_value(0x01) == 2.0 ** -9


def test_e8m0_decode_matches_torch_float8_e8m0fnu():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    ours = np.array([oracle.e8m0_value(b) for b in range(256)])
    assert np.isnan(ref[255]) and np.isnan(ours[255])
    assert np.array_equal(ref[:255], ours[:255])
    # closed form 2^(b-127)
    assert all(ours[b] == math.ldexp(1.0, b - 127) for b in range(255))


def test_bf16_decode_matches_bit_reinterpretation():
    bits = np.arange(65536, dtype=np.uint32)
    with np.errstate(invalid="ignore"):
        ref = (bits << 16).view(np.float32).astype(np.float64)
    ours = np.array([oracle.bf16_value(int(b)) for b in range(0, 65536, 7)])
    r = ref[::7]
    nan = np.isnan(r)
    assert np.array_equal(nan, np.isnan(ours))
    assert np.array_equal(r[~nan], ours[~nan])


def _e4m3_domain_values():
    """fp32 values in [-448, 448]: every bf16 pattern there, every exact midpoint
    between neighbouring e4m3 values and its fp32 neighbours, and random fp32."""
    bits = np.arange(65536, dtype=np.uint32) << 16
    vals = bits.view(np.float32)
    vals = vals[np.isfinite(vals) & (np.abs(vals) <= 448)]
    grid = np.array(sorted({abs(oracle.e4m3_value(b)) for b in range(0x7F)}), dtype=np.float64)
    mids = ((grid[1:] + grid[:-1]) / 2).astype(np.float32)  # exact in fp32
    near = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))])
    rng = np.random.default_rng(7)
    rnd = (rng.standard_normal(20000) * np.exp2(rng.integers(-12, 9, 20000))).astype(np.float32)
    rnd = rnd[np.abs(rnd) <= 448]
    allv = np.concatenate([vals, near, -near, rnd])
    return allv[np.abs(allv) <= 448]


def test_e4m3_encode_matches_torch_rne_in_range():
    v = _e4m3_domain_values()
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = oracle.e4m3_encode(v)
    bad = np.nonzero(ref != ours)[0]
    assert bad.size == 0, [(float(v[i]), hex(ref[i]), hex(ours[i])) for i in bad[:10]]


def test_e4m3_encode_saturates_and_nan():
    v = np.array([448.0, 449.0, 464.0, 500.0, 1e30, np.inf, -449.0, -np.inf], np.float32)
    assert list(oracle.e4m3_encode(v)) == [0x7E] * 6 + [0xFE] * 2
    assert oracle.e4m3_encode(np.array([np.nan], np.float32))[0] == 0x7F
    assert oracle.e4m3_encode(np.array([-0.0], np.float32))[0] == 0x80


def test_e2m1_encode_hand_worked_points():
    pts = e2m1_points()
    v = np.array([p[0] for p in pts], np.float32)
    for (x, want), x32 in zip(pts, v):
        if abs(x) not in (6.0001, 1e9, 1e-30):
            assert float(x32) == x  # fixture values are exact fp32
    got = oracle.e2m1_encode(v)
    for (x, want), g in zip(pts, got):
        assert g == want, (x, hex(want), hex(int(g)))


def test_e2m1_encode_is_nearest_even_on_a_dense_sweep():
    # Brute force: nearest of the 8 listed magnitudes, ties to the even code.
    x = np.linspace(-7, 7, 28001, dtype=np.float32)
    got = oracle.e2m1_encode(x)
    for xi, g in zip(x, got):
        a = abs(float(xi))
        d = [abs(m - a) for m in E2M1_LISTED]
        best = min(range(8), key=lambda c: (d[c], c & 1))
        if a >= 6:
            best = 7
        want = best | (8 if math.copysign(1, float(xi)) < 0 else 0)
        assert g == want, (float(xi), g, want)


def _bf16_nearest_even(y: float) -> int:
    """Independent bf16 rounding (normal range): 8 significant bits, Python's
    exact round-half-even on the scaled significand."""
    if y == 0:
        return 0x8000 if math.copysign(1, y) < 0 else 0
    f, e = math.frexp(abs(y))  # |y| = f * 2^e, f in [0.5, 1)
    q = round(Fraction(f) * 256)  # Fraction rounding is exact half-even
    val = math.ldexp(float(q), e - 8)
    bits = int(np.array([val], np.float32).view(np.uint32)[0]) >> 16
    return bits | (0x8000 if y < 0 else 0)


def test_bf16_round_matches_exact_half_even():
    rng = np.random.default_rng(3)
    y = rng.standard_normal(5000) * np.exp2(rng.integers(-60, 60, 5000))
    # exact bf16 midpoints and their double neighbours
    b = (rng.integers(0x0080, 0x7F00, 2000).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ulp = np.exp2(np.floor(np.log2(b)) - 7)
    mids = b + ulp / 2
    y = np.concatenate([y, mids, np.nextafter(mids, 0), np.nextafter(mids, np.inf), -mids])
    got = oracle.bf16_round(y)
    for yi, g in zip(y, got):
        assert g == _bf16_nearest_even(float(yi)), (yi, hex(int(g)))


_OVF = math.ldexp(1.0, 128) * (1 - 2.0 ** -9)  # midpoint between the largest bf16 and 2^128


@pytest.mark.parametrize("y,bits", [(0.0, 0x0000), (-0.0, 0x8000), (1.0, 0x3F80), (np.inf, 0x7F80),
                                    (_OVF, 0x7F80), (float(np.nextafter(_OVF, 0)), 0x7F7F),
                                    (3.3895313892515355e38, 0x7F7F)])
def test_bf16_round_specials(y, bits):
    assert oracle.bf16_round(np.array([y]))[0] == bits
