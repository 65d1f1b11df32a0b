"""Pins for the oracle's block-scaled GEMM (decode + float64 contraction + epilogue).

The GEMM the pages call is ``mm_fp4(x_fp4, w_fp4.T, x_scale, w_scale.T, alpha,
bf16)`` then ``out + bias`` (hao-ai-lab-FastVideo nvfp4_qat_config.py,
``NVFP4QATQuantizeMethod.apply``), with alpha = 1/(gs_x*gs_w); the MXFP8 one is
``npu_quant_matmul`` with per-group e8m0 scales on both operands and a bias
(vllm-omni mxfp8_config.py, ``NPUMxfp8LinearMethod._quant_matmul``).  These
checks compare the oracle with brute force over all code pairs, an exact int64
matmul, and torch's float8 decoders.
"""
import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_05_b200 import workloads as wl

E2M1_LISTED = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
ONE_E4M3 = 0x38  # 1.0
INT_CODES = {0: 0, 2: 1, 4: 2, 5: 3, 6: 4, 7: 6, 10: -1, 12: -2, 13: -3, 14: -4, 15: -6, 8: 0}


def _pack(codes: np.ndarray) -> np.ndarray:
    """[R, K] nibble codes -> [R, K/2] bytes, element 2j in the low nibble."""
    c = codes.astype(np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def _sf_buffer(rows, K, group, byte_of):
    cols = K // group
    cols_p = -(-cols // 4) * 4
    sf = np.zeros(oracle.sf_bytes(rows, cols), np.uint8)
    for r in range(rows):
        for c in range(cols):
            sf[oracle.sf_offset(r, c, cols_p)] = byte_of(r, c)
    return sf


def test_all_code_pairs_brute_force():
    """K = 16 GEMMs: row i of A holds code i everywhere, row j of B code j; scales 1."""
    K = 16
    A = _pack(np.repeat(np.arange(16)[:, None], K, 1))
    B = _pack(np.repeat(np.arange(16)[:, None], K, 1))
    sfA = _sf_buffer(16, K, 16, lambda r, c: ONE_E4M3)
    sfB = _sf_buffer(16, K, 16, lambda r, c: ONE_E4M3)
    decA = oracle.nvfp4_dequantize(A, sfA, K)
    decB = oracle.nvfp4_dequantize(B, sfB, K)
    y, bound = oracle.linear_reference(decA, decB)
    for i in range(16):
        for j in range(16):
            vi = -E2M1_LISTED[i & 7] if i & 8 else E2M1_LISTED[i & 7]
            vj = -E2M1_LISTED[j & 7] if j & 8 else E2M1_LISTED[j & 7]
            assert y[i, j] == 16 * vi * vj
            assert bound[i, j] == 16 * abs(vi * vj)


def test_integer_codes_unit_scales_equal_int64_matmul():
    rng = np.random.default_rng(1)
    M, N, K = 37, 29, 512
    keys = np.array(list(INT_CODES))
    ca = keys[rng.integers(0, keys.size, (M, K))]
    cb = keys[rng.integers(0, keys.size, (N, K))]
    ia = np.vectorize(INT_CODES.get)(ca).astype(np.int64)
    ib = np.vectorize(INT_CODES.get)(cb).astype(np.int64)
    sfA = _sf_buffer(M, K, 16, lambda r, c: ONE_E4M3)
    sfB = _sf_buffer(N, K, 16, lambda r, c: ONE_E4M3)
    y, _ = oracle.linear_reference(oracle.nvfp4_dequantize(_pack(ca), sfA, K),
                                   oracle.nvfp4_dequantize(_pack(cb), sfB, K))
    assert np.array_equal(y, (ia @ ib.T).astype(np.float64))


def test_power_of_two_group_scales_equal_shifted_int_matmul():
    """Per-group scales 2^s (e4m3 bytes of powers of two) -- the scale of group g
    multiplies exactly that group's partial product."""
    rng = np.random.default_rng(2)
    M, N, K = 9, 11, 256
    G = K // 16
    keys = np.array(list(INT_CODES))
    ca = keys[rng.integers(0, keys.size, (M, K))]
    cb = keys[rng.integers(0, keys.size, (N, K))]
    ia = np.vectorize(INT_CODES.get)(ca).astype(np.int64)
    ib = np.vectorize(INT_CODES.get)(cb).astype(np.int64)
    sa = rng.integers(-6, 8, (M, G))  # e4m3 normal powers of two: byte (s+7)<<3
    sb = rng.integers(-6, 8, (N, G))
    sfA = _sf_buffer(M, K, 16, lambda r, c: (int(sa[r, c]) + 7) << 3)
    sfB = _sf_buffer(N, K, 16, lambda r, c: (int(sb[r, c]) + 7) << 3)
    y, _ = oracle.linear_reference(oracle.nvfp4_dequantize(_pack(ca), sfA, K),
                                   oracle.nvfp4_dequantize(_pack(cb), sfB, K))
    ref = np.zeros((M, N), np.float64)
    for g in range(G):
        part = ia[:, g * 16:(g + 1) * 16] @ ib[:, g * 16:(g + 1) * 16].T
        ref += part.astype(np.float64) * np.exp2(sa[:, g][:, None] + sb[:, g][None, :])
    assert np.array_equal(y, ref)


def test_epilogue_alpha_row_scale_bias():
    rng = np.random.default_rng(3)
    decA = rng.integers(-6, 7, (5, 32)).astype(np.float64)
    decB = rng.integers(-6, 7, (7, 32)).astype(np.float64)
    bias = wl.normal_bf16(rng, (7,), 0.5)
    rs = np.array([1.0, 0.5, 2.0, 0.25, 3.0], np.float32)
    y, bound = oracle.linear_reference(decA, decB, alpha=0.375, row_scale=rs, bias=bias)
    acc = (decA.astype(np.int64) @ decB.astype(np.int64).T).astype(np.float64)
    want = 0.375 * rs.astype(np.float64)[:, None] * acc + wl.bf16_bits_to_f32(bias).astype(np.float64)
    assert np.array_equal(y, want)
    assert np.array_equal(bound, 0.375 * rs.astype(np.float64)[:, None] *
                          (np.abs(decA) @ np.abs(decB).T))


def test_nibble_order_low_nibble_is_even_k():
    codes = np.zeros((1, 32), np.int64)
    codes[0, 0] = 2   # 1.0 at k = 0 (low nibble of byte 0)
    codes[0, 1] = 7   # 6.0 at k = 1 (high nibble of byte 0)
    packed = _pack(codes)
    assert packed[0, 0] == 0x72
    dec = oracle.nvfp4_dequantize(packed, _sf_buffer(1, 32, 16, lambda r, c: ONE_E4M3), 32)
    assert dec[0, 0] == 1.0 and dec[0, 1] == 6.0 and np.all(dec[0, 2:] == 0)


def test_scale_lookup_uses_the_tile_map():
    """One scale byte set to 2.0 changes exactly one row-group of the decode."""
    M, K = 200, 128
    codes = np.full((M, K // 2), 0x22, np.uint8)  # every element 1.0
    target = (150, 5)
    sf = _sf_buffer(M, K, 16, lambda r, c: 0x40 if (r, c) == target else ONE_E4M3)
    dec = oracle.nvfp4_dequantize(codes, sf, K)
    want = np.ones((M, K))
    want[150, 80:96] = 2.0
    assert np.array_equal(dec, want)


def test_mxfp8_decode_matches_torch_float8_types():
    rng = np.random.default_rng(6)
    M, K = 130, 96
    q = rng.integers(0, 256, (M, K)).astype(np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x11  # no NaN codes
    e = rng.integers(100, 150, (M, K // 32))
    sf = _sf_buffer(M, K, 32, lambda r, c: int(e[r, c]))
    dec = oracle.mxfp8_dequantize(q, sf, K)
    tq = torch.from_numpy(q).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ts = torch.from_numpy(e.astype(np.uint8)).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    want = tq * np.repeat(ts, 32, axis=1)
    assert np.array_equal(dec, want)


def test_quantized_linear_approximates_the_bf16_linear():
    """End to end on the tiny workload: NVFP4 W4A4 stays within the format's
    error of the unquantized product (sanity, not a parity bound)."""
    lin = wl.tiny()
    gs_w = oracle.nvfp4_global_scale(oracle.amax_bf16(lin.W))
    ca, sa = oracle.nvfp4_quantize(lin.A, 1.0)
    cb, sb = oracle.nvfp4_quantize(lin.W, gs_w)
    alpha = np.float32(1.0) / (np.float32(1.0) * gs_w)
    y, _ = oracle.linear_reference(oracle.nvfp4_dequantize(ca, sa, lin.K),
                                   oracle.nvfp4_dequantize(cb, sb, lin.K), alpha=alpha)
    ref = wl.bf16_bits_to_f32(lin.A).astype(np.float64) @ wl.bf16_bits_to_f32(lin.W).astype(np.float64).T
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert 0.02 < rel < 0.2
