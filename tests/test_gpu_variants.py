"""Variants of the NVFP4 path on the GPU vs the oracle: the 4over6 global
scale numerator (sgl-project sglang nvfp4_online.py, _quantize_weight_nvfp4:
e4m3_max = 256), one scale shared by a gated w1/w3 pair (the same file,
process_loaded_weight), and fp16 input (hao-ai-lab-FastVideo nvfp4_config.py,
_coerce_fp4_input_dtype).  Scales, codes and scale bytes bit-exact; GEMMs
within the tolerance of tests/_gpu.py."""
import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_05_b200 import api
from block_scaled_precision_05_b200 import workloads as wl
from tests._gpu import DEV, assert_gemm_close, down, up_bf16

pytestmark = pytest.mark.gpu


def _bf16(rows, K, seed, std=1.0):
    rng = np.random.default_rng(seed)
    return wl.f32_to_bf16_bits((rng.standard_normal((rows, K)) * std).astype(np.float32))


AMAXES = [0.0, 1e-30, 2.0 ** -130, 0.02, 0.0625, 1.0, 3.0, 6.0, 447.0, 1536.0, 3.0e38]


@pytest.mark.parametrize("fmax", [api.FP8_FP4_MAX, api.FP8_FP4_MAX_4OVER6, 1000.0])
def test_global_scale_matches_oracle(fmax):
    for a in AMAXES:
        t = torch.tensor([a], dtype=torch.float32, device=DEV)
        gs, inv = api.nvfp4_global_scale(t, fmax)
        g_ref = oracle.nvfp4_global_scale(np.float32(a), fmax)
        assert down(gs)[0] == g_ref, (a, fmax)
        assert down(inv)[0] == np.float32(1.0) / g_ref, (a, fmax)


def test_amax_into_is_the_joint_amax():
    w1, w3 = _bf16(300, 256, seed=31, std=0.02), _bf16(200, 256, seed=32, std=0.07)
    a = api.amax(up_bf16(w1))
    api.amax_into(up_bf16(w3), a)
    ref = oracle.amax_bf16(np.concatenate([w1, w3]))
    assert down(a)[0] == np.float32(ref)
    b = api.amax(up_bf16(w3))
    api.amax_into(up_bf16(w1), b)  # order does not matter
    assert down(b)[0] == down(a)[0]


def test_shared_scale_quantization_bit_exact():
    w1, w3 = _bf16(256, 512, seed=33, std=0.02), _bf16(384, 512, seed=34, std=0.05)
    (q1, q3), gs, inv = api.nvfp4_quantize_shared([up_bf16(w1), up_bf16(w3)])
    g_ref = oracle.nvfp4_global_scale(oracle.amax_bf16(np.concatenate([w1, w3])))
    assert down(gs)[0] == g_ref
    for q, w in ((q1, w1), (q3, w3)):
        c, s = oracle.nvfp4_quantize(w, g_ref)
        assert np.array_equal(down(q.codes), c)
        assert np.array_equal(down(q.sf), s)
    # the same bytes as quantizing the concatenation and splitting it
    qc = api.nvfp4_quantize(up_bf16(np.concatenate([w1, w3])), gs)
    assert torch.equal(qc.codes, torch.cat([q1.codes, q3.codes]))
    assert torch.equal(qc.sf, torch.cat([q1.sf, q3.sf]))
    assert api.device_status() == 0


def test_four_over_six_weight_scales_and_gemm():
    M, N, K = 300, 384, 1024
    A, W = _bf16(M, K, seed=35), _bf16(N, K, seed=36, std=0.02)
    bias = _bf16(1, N, seed=37, std=0.01)[0]
    layer = api.NVFP4Linear(up_bf16(W), up_bf16(bias), four_over_six=True)
    g_ref = oracle.nvfp4_global_scale(oracle.amax_bf16(W), 1536.0)
    assert down(layer.gs_w)[0] == g_ref
    cb, sb = oracle.nvfp4_quantize(W, g_ref)
    assert np.array_equal(down(layer.weight.codes), cb)
    assert np.array_equal(down(layer.weight.sf), sb)
    assert down(layer.weight.sf).max() == 0x78  # e4m3 256: the 4over6 ceiling
    D = layer(up_bf16(A))
    assert api.device_status() == 0
    ca, sa = oracle.nvfp4_quantize(A, np.float32(1.0))
    decA, decB = oracle.nvfp4_dequantize(ca, sa, K), oracle.nvfp4_dequantize(cb, sb, K)
    alpha = np.float32(1) / (np.float32(1) * g_ref)
    ref, bound = oracle.linear_reference(decA, decB, alpha=alpha, row_scale=None, bias=bias)
    assert_gemm_close(D, ref, bound, "4over6 linear")


@pytest.mark.parametrize("per_token", [False, True])
def test_shared_scale_group_layers(per_token):
    M, N, K = 200, 256, 768
    A = _bf16(M, K, seed=38)
    w1, w3 = _bf16(N, K, seed=39, std=0.02), _bf16(N, K, seed=40, std=0.03)
    l1, l3 = api.NVFP4Linear.shared_scale_group([up_bf16(w1), up_bf16(w3)], per_token=per_token)
    assert torch.equal(l1.gs_w, l3.gs_w)
    g_ref = oracle.nvfp4_global_scale(oracle.amax_bf16(np.concatenate([w1, w3])))
    assert down(l1.gs_w)[0] == g_ref
    x = up_bf16(A)
    if per_token:
        gs_rows, inv_rows = oracle.row_global_scales(A)
        ca, sa = oracle.nvfp4_quantize(A, gs_rows, per_row=True)
        alpha, rs = np.float32(1) / g_ref, inv_rows
    else:
        ca, sa = oracle.nvfp4_quantize(A, np.float32(1.0))
        alpha, rs = np.float32(1) / (np.float32(1) * g_ref), None
    decA = oracle.nvfp4_dequantize(ca, sa, K)
    for layer, w in ((l1, w1), (l3, w3)):
        D = layer(x)
        cb, sb = oracle.nvfp4_quantize(w, g_ref)
        ref, bound = oracle.linear_reference(decA, oracle.nvfp4_dequantize(cb, sb, K), alpha=alpha, row_scale=rs,
                                             bias=None)
        assert_gemm_close(D, ref, bound, f"shared-scale layer per_token={per_token}")
    assert api.device_status() == 0


# --------------------------------------------------------------------------- fp16 input
def _f16(rows, K, seed, std=1.0, special=False):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((rows, K)) * std).astype(np.float16).view(np.uint16)
    if special and rows * K >= 64:
        flat = x.reshape(-1)
        n = flat.size
        flat[rng.integers(0, n, n // 20)] = 0x8000   # -0
        flat[rng.integers(0, n, n // 50)] = 0x0001   # smallest subnormal
        flat[rng.integers(0, n, n // 50)] = 0x8203   # negative subnormal
        flat[rng.integers(0, n, n // 100)] = 0x7BFF  # largest finite, 65504
        if K >= 32:
            x[0, :32] = 0
    return x


def _up_f16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.float16).to(DEV)


F16_SHAPES = [(1, 16), (7, 48), (129, 64), (300, 1536), (257, 5120), (64, 13824), (130, 80)]


@pytest.mark.parametrize("M,K", F16_SHAPES)
@pytest.mark.parametrize("per_row", [False, True])
def test_f16_quantize_bit_exact(M, K, per_row):
    x = _f16(M, K, seed=M * 3 + K, special=True)
    if per_row:
        q = api.nvfp4_quantize(_up_f16(x), per_row=True)
        gs, inv = oracle.row_global_scales(x, fmt="f16")
        assert np.array_equal(down(q.row_gs), gs) and np.array_equal(down(q.row_inv_gs), inv)
        codes, sf = oracle.nvfp4_quantize(x, gs, per_row=True, fmt="f16")
    else:
        g = np.float32(0.37109375)
        q = api.nvfp4_quantize(_up_f16(x), torch.tensor([g], device=DEV))
        codes, sf = oracle.nvfp4_quantize(x, g, fmt="f16")
    assert np.array_equal(down(q.codes), codes)
    assert np.array_equal(down(q.sf), sf)


def test_f16_amax():
    x = _f16(333, 520, seed=42, std=30.0, special=True)
    x[5, 7] = 0xFC00  # -inf -> 65504
    a = api.amax(_up_f16(x))
    assert down(a)[0] == np.float32(oracle.amax_f16(x))
    y = _f16(10, 64, seed=43)
    y[0, 0] = 0x7E00  # NaN counts as 0
    b = api.amax(_up_f16(y))
    assert down(b)[0] == np.float32(oracle.amax_f16(y))


@pytest.mark.parametrize("per_token", [False, True])
def test_f16_linear(per_token):
    M, N, K = 200, 512, 1536
    A, W = _f16(M, K, seed=44), _f16(N, K, seed=45, std=0.02)
    layer = api.NVFP4Linear(_up_f16(W), per_token=per_token)
    g_ref = oracle.nvfp4_global_scale(oracle.amax_f16(W))
    assert down(layer.gs_w)[0] == g_ref
    cb, sb = oracle.nvfp4_quantize(W, g_ref, fmt="f16")
    assert np.array_equal(down(layer.weight.codes), cb)
    D = layer(_up_f16(A))
    assert D.dtype == torch.bfloat16
    assert api.device_status() == 0
    if per_token:
        gs_rows, inv_rows = oracle.row_global_scales(A, fmt="f16")
        ca, sa = oracle.nvfp4_quantize(A, gs_rows, per_row=True, fmt="f16")
        alpha, rs = np.float32(1) / g_ref, inv_rows
    else:
        ca, sa = oracle.nvfp4_quantize(A, np.float32(1.0), fmt="f16")
        alpha, rs = np.float32(1) / (np.float32(1) * g_ref), None
    ref, bound = oracle.linear_reference(oracle.nvfp4_dequantize(ca, sa, K), oracle.nvfp4_dequantize(cb, sb, K),
                                         alpha=alpha, row_scale=rs, bias=None)
    assert_gemm_close(D, ref, bound, f"fp16 linear per_token={per_token}")
