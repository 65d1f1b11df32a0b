"""tcgen05 block-scaled GEMMs vs the oracle's float64 contraction.

Tolerance (tests/_gpu.py, gemm_tolerance): fp32 output within
1e-3 * |alpha * row_scale| * sum_k |a_k b_k| of the exact value; bf16 output
within that plus one bf16 ulp, and within one ulp of bf16(exact) wherever the
accumulation bound is below half an ulp.
"""
import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_05_b200 import api
from block_scaled_precision_05_b200 import workloads as wl
from tests._gpu import DEV, assert_gemm_close, band_rows, down, sample_bands, up, up_bf16

pytestmark = pytest.mark.gpu


def _nvfp4_case(A, W, bias=None, per_token=False, rows=None, out_dtype=torch.bfloat16):
    """Runs the NVFP4 linear on the GPU and the oracle; compares the chosen rows."""
    M, K = A.shape
    w = up_bf16(W)
    gs_w, inv_gs_w = api.nvfp4_global_scale(api.amax(w))
    wq = api.nvfp4_quantize(w, gs_w)
    if per_token:
        aq = api.nvfp4_quantize(up_bf16(A), per_row=True)
        alpha, row_scale = inv_gs_w, aq.row_inv_gs
    else:
        gs_x = torch.ones(1, device=DEV)
        aq = api.nvfp4_quantize(up_bf16(A), gs_x)
        alpha, row_scale = api.nvfp4_alpha(gs_x, gs_w), None
    b = None if bias is None else up_bf16(bias)
    D = api.nvfp4_gemm(aq, wq, alpha, row_scale, b, out_dtype=out_dtype)
    assert api.device_status() == 0

    # oracle, from the same bf16 inputs only
    gso = oracle.nvfp4_global_scale(oracle.amax_bf16(W))
    cb, sb = oracle.nvfp4_quantize(W, gso)
    rows = np.arange(M) if rows is None else np.asarray(rows)
    bands = sorted(set((rows // 128).tolist()))
    decA = np.zeros((rows.size, K))
    rs = None
    for b_ in bands:
        r0, r1 = b_ * 128, min(M, b_ * 128 + 128)
        sel = (rows >= r0) & (rows < r1)
        if per_token:
            gs, inv = oracle.row_global_scales(A[r0:r1])
            ca, sa = oracle.nvfp4_quantize(A[r0:r1], gs, per_row=True)
        else:
            ca, sa = oracle.nvfp4_quantize(A[r0:r1], 1.0)
        decA[sel] = oracle.nvfp4_dequantize(ca, sa, K, rows=rows[sel] - r0)
    if per_token:
        _, inv_all = oracle.row_global_scales(A[rows])
        rs = inv_all
        alpha_o = np.float32(1) / gso
    else:
        alpha_o = np.float32(1) / (np.float32(1) * gso)
    decB = oracle.nvfp4_dequantize(cb, sb, K)
    ref, bound = oracle.linear_reference(decA, decB, alpha=alpha_o, row_scale=rs, bias=bias)
    assert_gemm_close(D[torch.as_tensor(rows, device=DEV)], ref, bound, f"nvfp4 M={M} N={W.shape[0]} K={K}")
    return D


def _mxfp8_case(A, W, bias=None, rows=None, out_dtype=torch.bfloat16):
    M, K = A.shape
    aq = api.mxfp8_quantize(up_bf16(A))
    wq = api.mxfp8_quantize(up_bf16(W))
    D = api.mxfp8_gemm(aq, wq, None, None if bias is None else up_bf16(bias), out_dtype=out_dtype)
    assert api.device_status() == 0
    rows = np.arange(M) if rows is None else np.asarray(rows)
    qb, sfb = oracle.mxfp8_quantize(W)
    decA = np.zeros((rows.size, K))
    for b_ in sorted(set((rows // 128).tolist())):
        r0, r1 = b_ * 128, min(M, b_ * 128 + 128)
        sel = (rows >= r0) & (rows < r1)
        qa, sfa = oracle.mxfp8_quantize(A[r0:r1])
        decA[sel] = oracle.mxfp8_dequantize(qa, sfa, K, rows=rows[sel] - r0)
    ref, bound = oracle.linear_reference(decA, oracle.mxfp8_dequantize(qb, sfb, K), bias=bias)
    assert_gemm_close(D[torch.as_tensor(rows, device=DEV)], ref, bound, f"mxfp8 M={M} N={W.shape[0]} K={K}")
    return D


def _rand(M, N, K, seed, bias=True):
    rng = np.random.default_rng(seed)
    A = wl.normal_bf16(rng, (M, K), outliers=True)
    W = wl.normal_bf16(rng, (N, K), 1.0 / np.sqrt(K))
    b = wl.normal_bf16(rng, (N,), 0.05) if bias else None
    return A, W, b


SHAPES = [(128, 256, 256), (1, 256, 256), (7, 8, 32), (129, 136, 96), (300, 520, 1024), (257, 264, 320),
          (64, 512, 2048), (513, 1024, 64), (200, 256, 5120)]


def test_tiny_config_exact_layer():
    lin = wl.tiny()
    _nvfp4_case(lin.A, lin.W)
    _nvfp4_case(lin.A, lin.W, out_dtype=torch.float32)


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_nvfp4_gemm_shapes(M, N, K, out_dtype):
    A, W, b = _rand(M, N, K, seed=M + 3 * N + 7 * K)
    _nvfp4_case(A, W, bias=b, out_dtype=out_dtype)


@pytest.mark.parametrize("M,N,K", [(1, 256, 512), (16, 264, 256), (130, 512, 1024)])
def test_nvfp4_gemm_per_token(M, N, K):
    A, W, b = _rand(M, N, K, seed=M * 5 + N, bias=False)
    _nvfp4_case(A, W, per_token=True, out_dtype=torch.float32)
    _nvfp4_case(A, W, bias=b, per_token=True)


@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (7, 8, 32), (129, 136, 96), (300, 520, 1024), (65, 264, 5120)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_mxfp8_gemm_shapes(M, N, K, out_dtype):
    A, W, b = _rand(M, N, K, seed=M + N + K)
    _mxfp8_case(A, W, bias=b, out_dtype=out_dtype)


# Shapes that take the CTA-pair form of the main kernel (M >= 512 and more
# 128 x 128 tiles than SMs): 256 x 256 tiles over two CTAs, each loading its
# 128 rows of A and half of B.  Ragged M where the second CTA's rows are all
# past M (600, 1000), N whose last tile leaves the second CTA's half of B past
# N (2568), a K tail shorter than a stage (352), several tiles per pair with
# more K stages than the ring (4096 x 4096 x 2048).
PAIR_SHAPES = [(600, 4096, 256), (1000, 2568, 352), (4096, 4096, 2048), (2100, 1536, 1536)]


@pytest.mark.parametrize("M,N,K", PAIR_SHAPES)
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_nvfp4_gemm_cta_pairs(M, N, K, out_dtype):
    A, W, b = _rand(M, N, K, seed=M + 3 * N + K)
    rows = None if M * N <= 4096 * 4096 else band_rows(M, sample_bands(M, 4, seed=1))
    _nvfp4_case(A, W, b, rows=rows, out_dtype=out_dtype)


@pytest.mark.parametrize("M,N,K", [(1100, 2304, 1024), (640, 4104, 512)])
def test_nvfp4_gemm_cta_pairs_per_token(M, N, K):
    A, W, b = _rand(M, N, K, seed=M + N)
    _nvfp4_case(A, W, b, per_token=True)


@pytest.mark.parametrize("M,N,K", [(700, 4096, 256), (1030, 2568, 384)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_mxfp8_gemm_cta_pairs(M, N, K, out_dtype):
    A, W, b = _rand(M, N, K, seed=M + 7 * N + K)
    _mxfp8_case(A, W, b, out_dtype=out_dtype)


@pytest.mark.parametrize("M,N,K,kind", [(32760, 1536, 1536, "nvfp4"), (600, 4096, 256, "nvfp4"),
                                         (1100, 2304, 1024, "per_token"), (2100, 4096, 1024, "mxfp8")])
def test_cta_pair_gemm_relaunches_are_bit_identical(M, N, K, kind):
    """The pair form hands stage and accumulator phases from one CTA to the
    other; relaunched on the same inputs (back to back, no synchronisation in
    between) it must give the same bits every time."""
    g = torch.Generator(device=DEV)
    g.manual_seed(M + N + K)
    A = torch.randn((M, K), generator=g, device=DEV).to(torch.bfloat16)
    W = (torch.randn((N, K), generator=g, device=DEV) / K ** 0.5).to(torch.bfloat16)
    b = (torch.randn((N,), generator=g, device=DEV) * 0.01).to(torch.bfloat16)
    if kind == "mxfp8":
        layer = api.MXFP8Linear(W, b)
        aq = api.mxfp8_quantize(A)

        def run(out):
            return api.mxfp8_gemm(aq, layer.weight, None, layer.bias, out=out)
    else:
        layer = api.NVFP4Linear(W, b, per_token=kind == "per_token")
        aq = layer.quantize_input(A)
        rs = aq.row_inv_gs if kind == "per_token" else None

        def run(out):
            return api.nvfp4_gemm(aq, layer.weight, layer.alpha, rs, layer.bias, out=out)
    ref = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    run(ref)
    outs = [torch.full_like(ref, float("nan")) for _ in range(4)]
    for _ in range(8):
        for o in outs:
            run(o)
        torch.cuda.synchronize()
        assert all(torch.equal(o, ref) for o in outs)
        for o in outs:
            o.fill_(float("nan"))
    assert api.device_status() == 0


@pytest.mark.parametrize("M,N,K", [(600, 4096, 256), (300, 520, 1024)])  # CTA pairs; one CTA per tile
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_strided_output_without_alpha_or_bias(M, N, K, out_dtype):
    """D written into a column slice of a wider buffer (row stride N + 24):
    the columns past N keep their contents; alpha and bias absent (alpha 1)."""
    A, W, _ = _rand(M, N, K, seed=M * 3 + N, bias=False)
    w = up_bf16(W)
    gs_w, _ = api.nvfp4_global_scale(api.amax(w))
    wq = api.nvfp4_quantize(w, gs_w)
    aq = api.nvfp4_quantize(up_bf16(A), torch.ones(1, device=DEV))
    wide = torch.full((M, N + 24), float("nan"), dtype=out_dtype, device=DEV)
    D = api.nvfp4_gemm(aq, wq, None, None, None, out_dtype=out_dtype, out=wide[:, :N])
    assert api.device_status() == 0
    assert D.stride(0) == N + 24
    assert torch.isnan(wide[:, N:]).all()
    gso = oracle.nvfp4_global_scale(oracle.amax_bf16(W))
    cb, sb = oracle.nvfp4_quantize(W, gso)
    ca, sa = oracle.nvfp4_quantize(A, 1.0)
    ref, bound = oracle.linear_reference(oracle.nvfp4_dequantize(ca, sa, K), oracle.nvfp4_dequantize(cb, sb, K))
    assert_gemm_close(D, ref, bound, f"strided D, no alpha / bias, M={M}")


def test_one_hot_scale_through_the_tensor_core():
    """All codes 1.0 and all scales 1.0, except one scale byte of A set to 2.0:
    exactly the 16 products of that (row, group) double, so only that output row
    changes, by 16 per column.  Pins the 128x4 scale map as the tensor core reads
    it.  (Nibble order cannot be seen this way: both operands use the same
    packing, so swapping it permutes k in both and leaves every sum unchanged;
    the packing itself is pinned by the bit-exact quantizer parity.)"""
    M, N, K = 200, 264, 256
    cols4 = K // 16
    codes_a = torch.full((M, K // 2), 0x22, dtype=torch.uint8, device=DEV)
    codes_b = torch.full((N, K // 2), 0x22, dtype=torch.uint8, device=DEV)
    sfa = np.zeros(api.nvfp4_sf_bytes(M, K), np.uint8)
    sfb = np.zeros(api.nvfp4_sf_bytes(N, K), np.uint8)
    for r in range(M):
        for c in range(cols4):
            sfa[oracle.sf_offset(r, c, cols4)] = 0x38
    for r in range(N):
        for c in range(cols4):
            sfb[oracle.sf_offset(r, c, cols4)] = 0x38
    sfa[oracle.sf_offset(150, 5, cols4)] = 0x40
    a = api.NVFP4Tensor(codes_a, up(sfa), K)
    b = api.NVFP4Tensor(codes_b, up(sfb), K)
    D = down(api.nvfp4_gemm(a, b, out_dtype=torch.float32))
    want = np.full((M, N), float(K))
    want[150, :] += 16.0
    assert np.array_equal(D, want)


def test_empty_gemm_is_a_no_op():
    a = api.NVFP4Tensor(torch.empty((0, 32), dtype=torch.uint8, device=DEV),
                        torch.empty(0, dtype=torch.uint8, device=DEV), 64)
    b = api.NVFP4Tensor(torch.zeros((8, 32), dtype=torch.uint8, device=DEV),
                        torch.zeros(api.nvfp4_sf_bytes(8, 64), dtype=torch.uint8, device=DEV), 64)
    assert api.nvfp4_gemm(a, b).shape == (0, 8)


def test_linear_module_flattens_leading_dims():
    rng = np.random.default_rng(5)
    A = wl.normal_bf16(rng, (2 * 3 * 50, 256))
    W = wl.normal_bf16(rng, (136, 256), 0.05)
    bias = wl.normal_bf16(rng, (136,), 0.1)
    layer = api.NVFP4Linear(up_bf16(W), up_bf16(bias))
    y3 = layer(up_bf16(A).view(2, 3, 50, 256))
    assert y3.shape == (2, 3, 50, 136)
    y2 = layer(up_bf16(A))
    assert torch.equal(y3.reshape(-1, 136), y2)
    with pytest.raises(TypeError):
        layer(torch.ones((4, 256), dtype=torch.int32, device=DEV))
    y32 = layer(up_bf16(A).float())  # fp32 input is cast to bf16 first
    assert torch.equal(y32, y2)


# ------------------------------------------------------------------- full-size workloads
def test_wan13_projection_sampled_rows():
    lin = wl.wan13()
    rows = band_rows(lin.M, sample_bands(lin.M, 2, seed=3))
    _nvfp4_case(lin.A, lin.W, bias=lin.bias, rows=rows)


@pytest.mark.parametrize("name", ["wan14_in", "wan14_out"])
def test_wan14_ffn_sampled_rows(name):
    lin = getattr(wl, name)()
    rng = np.random.default_rng(9)
    rows = np.unique(np.concatenate([rng.integers(0, lin.M, 96), np.arange(lin.M - 40, lin.M)]))
    _nvfp4_case(lin.A, lin.W, rows=rows)


@pytest.mark.parametrize("M", wl.SKINNY_M)
def test_skinny_per_token_sweep(M):
    lin = wl.skinny(M)
    rows = np.arange(M) if M <= 128 else np.unique(np.random.default_rng(M).integers(0, M, 128))
    _nvfp4_case(lin.A, lin.W, per_token=True, rows=rows)


def test_mxfp8_config_sampled_rows():
    lin = wl.mxfp8()
    rng = np.random.default_rng(10)
    rows = np.unique(np.concatenate([rng.integers(0, lin.M, 96), np.arange(lin.M - 40, lin.M)]))
    _mxfp8_case(lin.A, lin.W, rows=rows)
