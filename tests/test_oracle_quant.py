"""Pins for the oracle's quantizers, global scales and the 128x4 scale map.

Sources: NVFP4 = e2m1 codes, group 16, e4m3 scales, fp32 global scale, scale
layout ``layout_128x4`` (hao-ai-lab-FastVideo nvfp4_config.py, module docstring
and ``_nvfp4_quantize``); weight global scale 448*6/amax (nvfp4_qat_config.py,
``convert_model_to_fp4``; the all-zero guard of sglang nvfp4_online.py,
``_quantize_weight_nvfp4``); MXFP8 = 32 elements per float8_e8m0fnu scale, OCP
MX (vllm-omni mxfp8_config.py, ``DiffusionMXFP8Config``).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_05_b200 import workloads as wl
from tests._golden import nvfp4_groups


def _bf16(vals):
    return wl.f32_to_bf16_bits(np.asarray(vals, np.float32))


def _group(x_bits, gs):
    """Quantize one 16-element group through the full-tensor entry (1 row, K=16)."""
    codes, sf = oracle.nvfp4_quantize(np.asarray(x_bits, np.uint16).reshape(1, 16), gs)
    c = []
    for b in codes[0]:
        c += [int(b) & 0xF, int(b) >> 4]
    return int(sf[0]), c


# ----------------------------------------------------------------------------- NVFP4 groups
@pytest.mark.parametrize("case", nvfp4_groups(), ids=lambda c: c[0])
def test_nvfp4_hand_worked_groups(case):
    name, gs, xs, want_sfb, want_codes = case
    sfb, codes = _group(_bf16(xs), gs)
    assert sfb == want_sfb, name
    assert codes == want_codes, name


def test_nvfp4_constructed_groups_roundtrip():
    """x_i = value(c_i) * sf / gs with a code of magnitude 6 present must quantize
    back to exactly (sfb, c_i) for every normal scale byte and power-of-two gs."""
    rng = np.random.default_rng(11)
    e2m1 = [oracle.e2m1_value(c) for c in range(16)]
    checked = 0
    for sfb in range(0x08, 0x7F):
        sf = oracle.e4m3_value(sfb)
        for gs in (1.0, 4.0, 0.125, 2.0 ** 10):
            codes = list(rng.integers(0, 16, 16))
            codes[int(rng.integers(0, 16))] = 7 if rng.random() < 0.5 else 15
            x = np.array([e2m1[c] * sf / gs for c in codes], np.float64)
            xb = _bf16(x)
            assert np.array_equal(wl.bf16_bits_to_f32(xb).astype(np.float64), x)  # exact inputs
            got_sfb, got_codes = _group(xb, gs)
            assert got_sfb == sfb
            # -0 (code 8) encodes back to 8, +0 to 0
            assert got_codes == [int(c) for c in codes], (sfb, gs)
            checked += 1
    assert checked == (0x7F - 0x08) * 4


def test_nvfp4_requantize_is_idempotent_for_normal_scales():
    """quant(dequant(quant(x))) == quant(x) when the group scale is a normal e4m3
    value and gs is a power of two (dequantized values are then exact bf16)."""
    rng = np.random.default_rng(5)
    M, K = 64, 256
    for gs in (1.0, 8.0, 1.0 / 8):
        x = wl.normal_bf16(rng, (M, K), std=3.0, outliers=True)
        codes, sf = oracle.nvfp4_quantize(x, gs)
        dec = oracle.nvfp4_dequantize(codes, sf, K) / gs
        cols_p = -(-(K // 16) // 4) * 4
        normal = np.array([[sf[oracle.sf_offset(m, c, cols_p)] >= 0x08 for c in range(K // 16)]
                           for m in range(M)])
        assert normal.mean() > 0.9
        xb = _bf16(dec)
        assert np.array_equal(wl.bf16_bits_to_f32(xb).astype(np.float64), dec)
        codes2, sf2 = oracle.nvfp4_quantize(xb, gs)
        for m in range(M):
            for c in range(K // 16):
                if not normal[m, c]:
                    continue
                o = oracle.sf_offset(m, c, cols_p)
                assert sf2[o] == sf[o]
                assert np.array_equal(codes2[m, c * 8:(c + 1) * 8], codes[m, c * 8:(c + 1) * 8])
        # the largest element of a normal-scale group always takes code 6 (+-7 / 15)
        for m in range(0, M, 7):
            for c in range(K // 16):
                if normal[m, c]:
                    nib = [int(b) & 0xF for b in codes[m, c * 8:(c + 1) * 8]] + \
                          [int(b) >> 4 for b in codes[m, c * 8:(c + 1) * 8]]
                    assert any(n & 7 == 7 for n in nib)


def test_nvfp4_per_row_equals_per_tensor_row_by_row():
    rng = np.random.default_rng(9)
    x = wl.normal_bf16(rng, (130, 64), outliers=True)
    gs, inv = oracle.row_global_scales(x)
    codes, sf = oracle.nvfp4_quantize(x, gs, per_row=True)
    cols_p = 4
    for m in (0, 1, 64, 127, 128, 129):
        c1, s1 = oracle.nvfp4_quantize(x[m:m + 1], gs[m])
        assert np.array_equal(codes[m], c1[0])
        assert [sf[oracle.sf_offset(m, c, cols_p)] for c in range(4)] == [s1[oracle.sf_offset(0, c, cols_p)] for c in range(4)]


def test_nvfp4_scale_padding_is_zero():
    rng = np.random.default_rng(2)
    M, K = 130, 80  # 5 scale columns -> padded to 8; rows padded to 256
    x = wl.normal_bf16(rng, (M, K))
    codes, sf = oracle.nvfp4_quantize(x, 1.0)
    assert sf.size == 256 * 8
    used = {oracle.sf_offset(m, c, 8) for m in range(M) for c in range(K // 16)}
    pad = np.array([i for i in range(sf.size) if i not in used])
    assert np.all(sf[pad] == 0)
    assert np.all(sf[sorted(used)] != 0)


def test_nvfp4_rejects_k_not_multiple_of_16():
    with pytest.raises(ValueError):
        oracle.nvfp4_quantize(np.zeros((2, 24), np.uint16), 1.0)


def _nibbles(codes):
    c = np.asarray(codes, np.uint8)
    return np.stack([c & 0xF, c >> 4], axis=-1).reshape(c.shape[0], -1)


def test_nvfp4_nan_products_encode_as_code_7():
    # NaN elements are left out of the group amax (6 here: scale byte 1.0,
    # decode factor 1) and written as code 7; the finite ones are unaffected
    x = _bf16([[3.0, -6.0, 0.5, 1.0] + [0.0] * 12])
    x[0, 2], x[0, 3] = 0x7FC1, 0xFFC3
    codes, sf = oracle.nvfp4_quantize(x, np.float32(1.0))
    assert sf[0] == 0x38
    assert list(_nibbles(codes)[0, :4]) == [5, 0xF, 7, 7]
    # a row whose amax (2^-133) is below 2688 / FLT_MAX: its scale is +inf,
    # the nonzero elements saturate to +-6 and the zeros (0 * inf) are code 7
    x = np.zeros((1, 16), np.uint16)
    x[0, 0], x[0, 1] = 0x0001, 0x8001
    gs, _ = oracle.row_global_scales(x)
    assert np.isinf(gs[0])
    codes, sf = oracle.nvfp4_quantize(x, gs, per_row=True)
    assert sf[0] == 0x7E  # fl32(2^-133 / 6) * inf = inf saturates to 448
    assert list(_nibbles(codes)[0]) == [7, 0xF] + [7] * 14


# ----------------------------------------------------------------------------- global scales
def test_weight_amax_ignores_nan_and_caps_inf():
    x = _bf16([1.0, -3.5, 2.0])
    assert oracle.amax_bf16(x) == 3.5
    nan = np.array([0x7FC0, 0x3F80], np.uint16)  # NaN, 1.0
    assert oracle.amax_bf16(nan) == 1.0
    inf = np.array([0xFF80, 0x3F80], np.uint16)  # -inf, 1.0 -> largest finite bf16
    assert oracle.amax_bf16(inf) == float(wl.bf16_bits_to_f32(np.array([0x7F7F], np.uint16))[0])
    assert oracle.amax_bf16(np.zeros(5, np.uint16)) == 0.0


def test_global_scale_formula():
    for amax in (1.0, 0.07, 3.5, 1e-3, 2688.0, 123.456):
        a = np.float32(amax)
        assert oracle.nvfp4_global_scale(a) == np.float32(2688.0) / a  # IEEE fp32 division
    assert oracle.nvfp4_global_scale(0.0) == 1.0


def test_row_global_scales():
    x = _bf16([[1.5, -6.0, 0.0, 2.0], [0.0, 0.0, -0.0, 0.0], [448.0, 1.0, 1.0, 1.0]])
    gs, inv = oracle.row_global_scales(x)
    assert gs[0] == np.float32(2688) / np.float32(6) and gs[1] == 1.0 and gs[2] == np.float32(6.0)
    assert np.array_equal(inv, (np.float32(1) / gs).astype(np.float32))


# ----------------------------------------------------------------------------- MXFP8
def _floor_log2_from_bits(b: int) -> int:
    """floor(log2 |x|) of a nonzero finite bf16 read off its bit fields."""
    e = (b >> 7) & 0xFF
    m = b & 0x7F
    if e:
        return e - 127
    return m.bit_length() - 1 - 133


def test_mxfp8_scale_exponent_from_bit_fields():
    rng = np.random.default_rng(4)
    x = wl.normal_bf16(rng, (8, 32 * 64), std=1.0)
    # widen the exponent range: scale each group by 2^k (k from -140 to +120), exact in bf16
    f = wl.bf16_bits_to_f32(x).astype(np.float64).reshape(8, 64, 32)
    k = rng.integers(-140, 121, (8, 64, 1))
    f = f * np.exp2(k.astype(np.float64))
    f[0, 0] = 0.0
    xb = _bf16(f.reshape(8, -1).astype(np.float32))
    q, sf = oracle.mxfp8_quantize(xb)
    cols_p = 64
    for m in range(8):
        for g in range(64):
            grp = xb[m, g * 32:(g + 1) * 32]
            mags = grp & 0x7FFF
            amax_bits = int(mags.max())
            if amax_bits == 0:
                want = 0
            else:
                want = min(max(_floor_log2_from_bits(amax_bits) - 8, -127), 127) + 127
            assert sf[oracle.sf_offset(m, g, cols_p)] == want


def test_mxfp8_elements_match_torch_e4m3_of_exactly_scaled_values():
    rng = np.random.default_rng(8)
    x = wl.normal_bf16(rng, (33, 256), outliers=True)
    q, sf = oracle.mxfp8_quantize(x)
    cols_p = 8
    xf = wl.bf16_bits_to_f32(x).astype(np.float64)
    for m in range(33):
        for g in range(8):
            e = int(sf[oracle.sf_offset(m, g, cols_p)]) - 127
            v = np.clip(xf[m, g * 32:(g + 1) * 32] * 2.0 ** (-e), -448, 448).astype(np.float32)
            ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            assert np.array_equal(q[m, g * 32:(g + 1) * 32], ref)
            assert np.abs(xf[m, g * 32:(g + 1) * 32]).max() * 2.0 ** (-e) >= 256  # top binade used


def test_mxfp8_zero_group_and_powers_of_two_exact():
    x = np.zeros((1, 64), np.uint16)
    x[0, 1] = 0x8000  # -0
    vals = [2.0 ** k for k in range(-5, 3)] * 4
    x[0, 32:] = _bf16(vals)
    q, sf = oracle.mxfp8_quantize(x)
    assert sf[oracle.sf_offset(0, 0, 4)] == 0 and q[0, 0] == 0 and q[0, 1] == 0x80
    deq = oracle.mxfp8_dequantize(q, sf, 64)
    assert np.array_equal(deq[0, 32:], np.array(vals))  # powers of two are exact
    assert sf[oracle.sf_offset(0, 1, 4)] == (2 - 8) + 127


# ----------------------------------------------------------------------------- 128x4 scale map
def test_sf_map_is_a_bijection_onto_the_padded_buffer():
    for rows, cols in ((1, 1), (128, 4), (130, 5), (300, 16), (256, 96)):
        rp, cp = -(-rows // 128) * 128, -(-cols // 4) * 4
        offs = np.array([oracle.sf_offset(r, c, cp) for r in range(rp) for c in range(cp)])
        assert offs.min() == 0 and offs.max() == rp * cp - 1
        assert np.unique(offs).size == rp * cp
        assert oracle.sf_bytes(rows, cols) == rp * cp


def test_sf_map_matches_blocked_reshape_formulation():
    """The tile map, written as the reshape/transposition that cuts a padded
    [R, C] scale matrix into 128x4 tiles whose 128 rows are interleaved as
    4 groups of 32 (each 16-byte line holds rows r, r+32, r+64, r+96)."""
    R, C = 384, 12
    lin = np.arange(R * C).reshape(R, C)
    blocked = lin.reshape(R // 128, 4, 32, C // 4, 4).transpose(0, 3, 2, 1, 4).reshape(-1)
    placed = np.empty(R * C, np.int64)
    for r in range(R):
        for c in range(C):
            placed[oracle.sf_offset(r, c, C)] = lin[r, c]
    assert np.array_equal(placed, blocked)
