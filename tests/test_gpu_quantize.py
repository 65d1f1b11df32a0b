"""NVFP4 / MXFP8 quantize kernels and the global-scale kernels vs the CPU oracle:
bit-exact codes, scale bytes (including padding) and per-row scales."""
import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_05_b200 import api
from block_scaled_precision_05_b200 import workloads as wl
from tests._gpu import DEV, band_rows, down, sample_bands, up, up_bf16

pytestmark = pytest.mark.gpu


def _data(M, K, seed, kind="normal"):
    rng = np.random.default_rng(seed)
    x = wl.normal_bf16(rng, (M, K), std=2.0, outliers=True)
    if kind == "special" and M * K >= 64:
        flat = x.reshape(-1)
        n = flat.size
        flat[rng.integers(0, n, n // 20)] = 0x8000              # -0
        flat[rng.integers(0, n, n // 50)] = 0x0001              # smallest subnormal
        flat[rng.integers(0, n, n // 50)] = 0x8003              # negative subnormal
        flat[rng.integers(0, n, n // 100)] = 0x7F7F             # largest finite
        if K >= 32:
            x[0, :32] = 0                                       # all-zero groups
            x[min(1, M - 1), :16] = wl.f32_to_bf16_bits(np.full(16, 1e-6, np.float32))  # scale underflow
    return x


SHAPES = [(1, 16), (1, 64), (7, 48), (128, 256), (129, 64), (130, 80), (300, 1536), (257, 5120), (64, 13824)]

# Dispatch branches of the quantize launchers (each instantiated for bf16 and
# fp16 input and for 128x4 and 8x4 scale tiles) and the bit-exact tests that
# reach each of them:
#
# nvfp4_quantize / _f16 / _ex (run_nvfp4_quantize):
#   per-row, K == 1024 / 1536 / 2048 / 5120 (any M)
#       nvfp4_quant_rowreg_kernel<G>    test_nvfp4_quantize_per_row_bit_exact (1536, 5120),
#                                       test_dispatch_branch_bit_exact[rowreg-*] (M 1 to 4100)
#   other K % 64 == 0, per-row, round_up(M) <= resident blocks (at most 148 x 8)
#       nvfp4_quant_rowblock_kernel     test_nvfp4_quantize_per_row_bit_exact (K 64, 256, 13824),
#                                       test_dispatch_branch_bit_exact[rowblock-*]
#   other K % 64 == 0, per-row, more rows
#       nvfp4_quant_k64_kernel<true>    test_dispatch_branch_bit_exact[k64-per-row-*] (M 2000, 4100)
#   per-tensor, K == 1024
#       nvfp4_quant_short_kernel<S=2>   test_dispatch_branch_bit_exact[short-1024-*]
#   per-tensor, K == 1536
#       nvfp4_quant_short_kernel<S=3>   test_nvfp4_quantize_per_tensor_bit_exact (300, 1536),
#                                       test_dispatch_branch_bit_exact[short-1536-*]
#   per-tensor, other K % 64 == 0
#       nvfp4_quant_k64_kernel<false>   test_nvfp4_quantize_per_tensor_bit_exact (K 64, 256, 5120, 13824)
#   K % 64 != 0 (per-tensor / per-row)
#       nvfp4_quant_generic_kernel      both SHAPES tests at K = 16, 48, 80
# nvfp4_rmsnorm_quantize (tests/test_gpu_rmsnorm.py):
#   K == 1536 / 2048                    nvfp4_rmsnorm_quant_short_kernel<per_row, S=3 / 4>
#   other K                             nvfp4_rmsnorm_quant_kernel<per_row>
# mxfp8_quantize:
#   K % 128 == 0                        mxfp8_quant_k128_kernel   test_mxfp8_quantize_bit_exact (K 128, 5120, 13824)
#   other K % 32 == 0                   mxfp8_quant_generic_kernel test_mxfp8_quantize_bit_exact (K 32, 96, 160)
BRANCH_CASES = [
    # (name, M, K, per_row)
    ("short-1024", 1, 1024, False), ("short-1024", 129, 1024, False), ("short-1024", 300, 1024, False),
    ("short-1024", 4100, 1024, False), ("short-1536", 4100, 1536, False),
    # rowreg: every (groups a thread G, warps a row S) the launcher picks
    ("rowreg", 1, 1024, True), ("rowreg", 4100, 1024, True),          # G1 S2, G2 S1
    ("rowreg", 1030, 1536, True), ("rowreg", 2000, 1536, True),       # G1 S3, G3 S1
    ("rowreg", 129, 2048, True), ("rowreg", 1000, 2048, True), ("rowreg", 4100, 2048, True),  # S4, S2, S1
    ("rowreg", 129, 5120, True), ("rowreg", 4100, 5120, True),        # G2 S5, G5 S2
    ("rowblock", 129, 3072, True), ("rowblock", 300, 13824, True),
    ("k64-per-row", 4100, 3072, True), ("k64-per-row", 2000, 4096, True),
]


def _f16_bits(M, K, seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((M, K)) * 3.0).astype(np.float32)
    x[rng.random((M, K)) < 0.001] *= 50.0
    bits = x.astype(np.float16).view(np.uint16)
    flat = bits.reshape(-1)
    flat[rng.integers(0, flat.size, flat.size // 50)] = 0x8203  # negative subnormal
    flat[rng.integers(0, flat.size, flat.size // 200)] = 0x7BFF  # 65504
    return bits


@pytest.mark.parametrize("name,M,K,per_row", BRANCH_CASES, ids=[f"{c[0]}-{c[1]}x{c[2]}" for c in BRANCH_CASES])
@pytest.mark.parametrize("fmt", ["bf16", "f16"])
@pytest.mark.parametrize("layout", ["128x4", "8x4"])
def test_dispatch_branch_bit_exact(name, M, K, per_row, fmt, layout):
    seed = M * 13 + K + (7 if fmt == "f16" else 0)
    if fmt == "f16":
        x = _f16_bits(M, K, seed)
        xt = torch.from_numpy(np.ascontiguousarray(x)).view(torch.float16).to(DEV)
    else:
        x = _data(M, K, seed=seed, kind="special")
        xt = up_bf16(x)
    if per_row:
        q = api.nvfp4_quantize(xt, per_row=True, sf_layout=layout)
        gs, inv = oracle.row_global_scales(x, fmt=fmt)
        assert np.array_equal(down(q.row_gs).view(np.uint32), gs.view(np.uint32))
        assert np.array_equal(down(q.row_inv_gs).view(np.uint32), inv.view(np.uint32))
        codes, sf = oracle.nvfp4_quantize(x, gs, per_row=True, fmt=fmt, layout=layout)
    else:
        g = np.float32(0.37109375) if M % 2 else np.float32(291.5)
        q = api.nvfp4_quantize(xt, torch.tensor([g], device=DEV), sf_layout=layout)
        codes, sf = oracle.nvfp4_quantize(x, g, fmt=fmt, layout=layout)
    assert np.array_equal(down(q.codes), codes)
    assert np.array_equal(down(q.sf), sf)


@pytest.mark.parametrize("M,K", SHAPES)
@pytest.mark.parametrize("gs", [1.0, 0.37109375, 291.5])
def test_nvfp4_quantize_per_tensor_bit_exact(M, K, gs):
    x = _data(M, K, seed=M * 7 + K, kind="special")
    g = torch.tensor([gs], dtype=torch.float32, device=DEV)
    q = api.nvfp4_quantize(up_bf16(x), g)
    codes, sf = oracle.nvfp4_quantize(x, np.float32(gs))
    assert np.array_equal(down(q.codes), codes)
    assert np.array_equal(down(q.sf), sf)


@pytest.mark.parametrize("M,K", SHAPES)
def test_nvfp4_quantize_per_row_bit_exact(M, K):
    x = _data(M, K, seed=M + K * 3, kind="special")
    q = api.nvfp4_quantize(up_bf16(x), per_row=True)
    gs, inv = oracle.row_global_scales(x)
    codes, sf = oracle.nvfp4_quantize(x, gs, per_row=True)
    assert np.array_equal(down(q.row_gs).view(np.uint32), gs.view(np.uint32))
    assert np.array_equal(down(q.row_inv_gs).view(np.uint32), inv.view(np.uint32))
    assert np.array_equal(down(q.codes), codes)
    assert np.array_equal(down(q.sf), sf)


def _wide_range_rows(M, K, seed):
    """Rows scaled by powers of two across the whole bf16 range, so the
    per-row scale 2688 / amax runs from ~1e-35 to +inf (a row of the
    smallest subnormal), plus all-zero, all -0, +-inf and NaN rows."""
    rng = np.random.default_rng(seed)
    e = rng.integers(-150, 125, size=(M, 1)).astype(np.float64)
    x = (rng.standard_normal((M, K)) * np.exp2(e)).astype(np.float32)
    bits = wl.f32_to_bf16_bits(x)
    bits[0] = 0
    bits[1 % M] = 0
    bits[1 % M, 7] = 0x0001                      # amax 2^-133: gs overflows to +inf
    bits[2 % M] = 0x8000
    bits[3 % M, 5] = 0x7F80                      # +inf counts as the largest finite
    bits[4 % M, 16:32] = 0x7FC1                  # a NaN group
    bits[4 % M, 40:44] = 0xFFC3                  # negative NaNs among finite values
    bits[5 % M, :] = wl.f32_to_bf16_bits(np.full(K, 2.0 ** -126, np.float32))
    return bits


@pytest.mark.parametrize("K", [1024, 1536, 2048, 5120])
@pytest.mark.parametrize("M", [40, 3000])
def test_per_row_scales_across_the_range(M, K):
    """The per-token decode factors fl32(gs / e4m3) at the extremes of gs."""
    x = _wide_range_rows(M, K, seed=M + K)
    q = api.nvfp4_quantize(up_bf16(x), per_row=True)
    gs, inv = oracle.row_global_scales(x)
    assert np.isinf(gs[1 % M]) and gs.min() < 1e-30
    codes, sf = oracle.nvfp4_quantize(x, gs, per_row=True)
    assert np.array_equal(down(q.row_gs).view(np.uint32), gs.view(np.uint32))
    assert np.array_equal(down(q.row_inv_gs).view(np.uint32), inv.view(np.uint32))
    assert np.array_equal(down(q.codes), codes)
    assert np.array_equal(down(q.sf), sf)


def test_nvfp4_quantize_strided_rows_and_overwrites_stale_padding():
    M, K, ld = 100, 128, 192
    rng = np.random.default_rng(1)
    big = wl.normal_bf16(rng, (M, ld))
    xt = up_bf16(big)[:, :K]
    out = api.NVFP4Tensor(torch.empty((M, K // 2), dtype=torch.uint8, device=DEV),
                          torch.full((api.nvfp4_sf_bytes(M, K),), 0xAB, dtype=torch.uint8, device=DEV), K)
    q = api.nvfp4_quantize(xt, torch.ones(1, device=DEV), out=out)
    codes, sf = oracle.nvfp4_quantize(np.ascontiguousarray(big[:, :K]), 1.0)
    assert np.array_equal(down(q.codes), codes)
    assert np.array_equal(down(q.sf), sf)


@pytest.mark.parametrize("M,K", [(1, 32), (5, 96), (128, 128), (129, 160), (300, 5120), (33, 13824)])
def test_mxfp8_quantize_bit_exact(M, K):
    x = _data(M, K, seed=M * 11 + K, kind="special")
    q = api.mxfp8_quantize(up_bf16(x))
    qo, sfo = oracle.mxfp8_quantize(x)
    assert np.array_equal(down(q.q), qo)
    assert np.array_equal(down(q.sf), sfo)


def test_mxfp8_wide_exponent_range():
    rng = np.random.default_rng(4)
    f = wl.bf16_bits_to_f32(wl.normal_bf16(rng, (16, 32 * 40))).astype(np.float64).reshape(16, 40, 32)
    f = f * np.exp2(rng.integers(-140, 121, (16, 40, 1)).astype(np.float64))
    x = wl.f32_to_bf16_bits(f.reshape(16, -1).astype(np.float32))
    q = api.mxfp8_quantize(up_bf16(x))
    qo, sfo = oracle.mxfp8_quantize(x)
    assert np.array_equal(down(q.q), qo)
    assert np.array_equal(down(q.sf), sfo)


def test_amax_global_scale_alpha():
    rng = np.random.default_rng(2)
    for n in (1, 7, 1000, 1 << 20, (1 << 20) + 3):
        x = wl.normal_bf16(rng, (n,), 0.02)
        if n > 10:
            x[3] = 0x7FC0  # NaN -> 0
            x[5] = 0xFF80  # -inf -> largest finite
        a = api.amax(up_bf16(x))
        ao = oracle.amax_bf16(x)
        assert float(a.item()) == ao
        gs, inv = api.nvfp4_global_scale(a)
        assert down(gs).view(np.uint32)[0] == np.float32(oracle.nvfp4_global_scale(ao)).view(np.uint32)
        assert down(inv)[0] == np.float32(1) / np.float32(oracle.nvfp4_global_scale(ao))
    z = api.amax(up_bf16(np.zeros(64, np.uint16)))
    assert float(z.item()) == 0.0
    assert float(api.nvfp4_global_scale(z)[0].item()) == 1.0
    gx = torch.tensor([1.0], device=DEV)
    gw = torch.tensor([123.456], device=DEV)
    al = api.nvfp4_alpha(gx, gw)
    assert down(al)[0] == np.float32(1) / (np.float32(1) * np.float32(123.456))


def test_empty_input_is_a_no_op():
    x = torch.empty((0, 64), dtype=torch.bfloat16, device=DEV)
    q = api.nvfp4_quantize(x, torch.ones(1, device=DEV))
    assert q.codes.shape == (0, 32) and q.sf.numel() == 0
    m = api.mxfp8_quantize(x)
    assert m.q.shape == (0, 64)


# ------------------------------------------------------------------- full-size workloads
def _check_bands(x, q_gpu, gs, per_row, bands, kind="nvfp4"):
    """Oracle-quantize whole 128-row bands and compare codes and scale bytes."""
    M, K = x.shape
    cols4 = -(-(K // (16 if kind == "nvfp4" else 32)) // 4) * 4
    for b in bands:
        r0, r1 = b * 128, min(M, b * 128 + 128)
        xb = x[r0:r1]
        if kind == "nvfp4":
            g = gs[r0:r1] if per_row else gs
            codes, sf = oracle.nvfp4_quantize(xb, g, per_row=per_row)
            got_codes = down(q_gpu.codes[r0:r1])
        else:
            codes, sf = oracle.mxfp8_quantize(xb)
            got_codes = down(q_gpu.q[r0:r1])
        assert np.array_equal(got_codes, codes), f"band {b}"
        got_sf = down(q_gpu.sf[b * 128 * cols4:(b + 1) * 128 * cols4])
        assert np.array_equal(got_sf, sf), f"band {b} scales"


def test_wan13_activation_quantize_full():
    lin = wl.wan13()
    q = api.nvfp4_quantize(up_bf16(lin.A), torch.ones(1, device=DEV))
    codes, sf = oracle.nvfp4_quantize(lin.A, 1.0)
    assert np.array_equal(down(q.codes), codes)
    assert np.array_equal(down(q.sf), sf)


@pytest.mark.parametrize("name", ["wan14_in", "wan14_out"])
def test_wan14_activation_quantize_sampled_bands(name):
    lin = getattr(wl, name)()
    q = api.nvfp4_quantize(up_bf16(lin.A), torch.ones(1, device=DEV))
    _check_bands(lin.A, q, np.float32(1.0), False, sample_bands(lin.M, 6, seed=1))


@pytest.mark.parametrize("name", ["wan14_in", "wan14_out", "mxfp8"])
def test_weight_quantize_full(name):
    lin = getattr(wl, name)()
    w = up_bf16(lin.W)
    if name == "mxfp8":
        q = api.mxfp8_quantize(w)
        qo, sfo = oracle.mxfp8_quantize(lin.W)
        assert np.array_equal(down(q.q), qo) and np.array_equal(down(q.sf), sfo)
        return
    gs, _ = api.nvfp4_global_scale(api.amax(w))
    gso = oracle.nvfp4_global_scale(oracle.amax_bf16(lin.W))
    assert float(gs.item()) == float(gso)
    q = api.nvfp4_quantize(w, gs)
    codes, sf = oracle.nvfp4_quantize(lin.W, gso)
    assert np.array_equal(down(q.codes), codes)
    assert np.array_equal(down(q.sf), sf)


def test_mxfp8_activation_quantize_sampled_bands():
    lin = wl.mxfp8()
    q = api.mxfp8_quantize(up_bf16(lin.A))
    _check_bands(lin.A, q, None, False, sample_bands(lin.M, 6, seed=2), kind="mxfp8")


@pytest.mark.parametrize("M", wl.SKINNY_M)
def test_skinny_per_token_quantize(M):
    lin = wl.skinny(M)
    q = api.nvfp4_quantize(up_bf16(lin.A), per_row=True)
    gs, inv = oracle.row_global_scales(lin.A)
    codes, sf = oracle.nvfp4_quantize(lin.A, gs, per_row=True)
    assert np.array_equal(down(q.row_gs), gs) and np.array_equal(down(q.row_inv_gs), inv)
    assert np.array_equal(down(q.codes), codes)
    assert np.array_equal(down(q.sf), sf)
