"""The skinny-M GEMM with its K range split over a thread-block cluster (few
weight panels: the CTAs of a cluster each stream a slice of K, and rank 0 adds
the others' fp32 partials, in rank order, from their shared memory) against the
oracle's float64 contraction, within the GEMM tolerance of tests/_gpu.py; the
result does not depend on timing (two launches agree bit for bit)."""
import numpy as np
import pytest
import torch

from block_scaled_precision_05_b200 import api
from block_scaled_precision_05_b200 import workloads as wl
from tests._gpu import DEV, up_bf16
from tests.test_gpu_gemm import _mxfp8_case, _nvfp4_case, _rand

pytestmark = pytest.mark.gpu

# (M, N, K): few panels (N <= 9K) and long K, so that K is split over 2-4
# CTAs (at least 16 k-blocks of 256 elements per CTA); ragged N and K, M
# across the three activation widths
SPLIT_SHAPES = [(1, 5120, 13824), (16, 5120, 8192), (33, 1536, 12288), (48, 264, 16384), (5, 1024, 8192),
                (17, 136, 12320), (1, 128, 16384), (40, 2048, 8192)]


@pytest.mark.parametrize("M,N,K", SPLIT_SHAPES)
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_split_k_matches_oracle(M, N, K, out_dtype):
    A, W, b = _rand(M, N, K, seed=M * 13 + N + K)
    _nvfp4_case(A, W, bias=b, out_dtype=out_dtype)


@pytest.mark.parametrize("M,N,K", [(1, 5120, 13824), (16, 1536, 12288), (45, 520, 8192)])
def test_split_k_per_token(M, N, K):
    A, W, b = _rand(M, N, K, seed=M + N * 3 + K, bias=False)
    _nvfp4_case(A, W, per_token=True, out_dtype=torch.float32)
    _nvfp4_case(A, W, bias=b, per_token=True)


@pytest.mark.parametrize("M,N,K", [(1, 5120, 13824), (24, 1024, 8192), (7, 264, 4096)])
def test_split_k_mxfp8(M, N, K):
    A, W, b = _rand(M, N, K, seed=M + 2 * N + K)
    _mxfp8_case(A, W, bias=b)


@pytest.mark.parametrize("M", [1, 9, 40, 64])
def test_split_k_8x4_scales(M):
    N, K = 2048, 8192
    A, W, _ = _rand(M, N, K, seed=M + 77, bias=False)
    w = up_bf16(W)
    gs_w, _ = api.nvfp4_global_scale(api.amax(w))
    wq = api.nvfp4_quantize(w, gs_w)
    a8 = api.nvfp4_quantize(up_bf16(A), per_row=True, sf_layout="8x4")
    a128 = api.nvfp4_quantize(up_bf16(A), per_row=True)
    _, inv_w = api.nvfp4_global_scale(api.amax(w))
    d8 = api.nvfp4_gemm(a8, wq, inv_w, a8.row_inv_gs, None, out_dtype=torch.float32)
    d128 = api.nvfp4_gemm(a128, wq, inv_w, a128.row_inv_gs, None, out_dtype=torch.float32)
    assert api.device_status() == 0
    assert torch.equal(d8, d128)  # same scale values reach the tensor core, same split


def test_split_k_is_deterministic():
    A, W, b = _rand(8, 5120, 13824, seed=5)
    w = up_bf16(W)
    gs_w, _ = api.nvfp4_global_scale(api.amax(w))
    wq = api.nvfp4_quantize(w, gs_w)
    gs_x = torch.ones(1, device=DEV)
    aq = api.nvfp4_quantize(up_bf16(A), gs_x)
    alpha = api.nvfp4_alpha(gs_x, gs_w)
    outs = [api.nvfp4_gemm(aq, wq, alpha, None, up_bf16(b), out_dtype=torch.float32) for _ in range(4)]
    assert api.device_status() == 0
    for o in outs[1:]:
        assert torch.equal(o, outs[0])


@pytest.mark.parametrize("M", [1, 16, 48])
def test_fc_out_decode_sweep(M):
    lin = wl.skinny_out(M)
    _nvfp4_case(lin.A, lin.W, per_token=True, rows=np.arange(M))
