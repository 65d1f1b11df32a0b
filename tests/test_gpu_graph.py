"""The quantize -> GEMM sequence inside a captured CUDA graph, and launched
back to back on a stream, gives exactly the results of separate, synchronised
calls.

The GEMM kernels are launched with programmatic stream serialisation (their
set-up may overlap the previous kernel); these tests fail if any of them read
the quantized activation, its scales or the per-row scales before the producing
kernel has finished.  Each replay first overwrites the captured input buffer
with new data, so stale reads show up as mismatches.
"""
import numpy as np
import pytest
import torch

from block_scaled_precision_05_b200 import api
from tests._gpu import DEV

pytestmark = pytest.mark.gpu


def _inputs(M, N, K, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    A = [torch.randn((M, K), generator=g, device=DEV).to(torch.bfloat16) for _ in range(3)]
    W = (torch.randn((N, K), generator=g, device=DEV) / K ** 0.5).to(torch.bfloat16)
    bias = (torch.randn((N,), generator=g, device=DEV) * 0.01).to(torch.bfloat16)
    return A, W, bias


def _separate(layer, a):
    """Reference: every launch followed by a device synchronisation."""
    xq = layer.quantize_input(a)
    torch.cuda.synchronize()
    y = layer(a, pre_quantized=xq)
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("M,N,K,per_token", [(16, 1536, 1536, True), (1000, 1536, 1536, False),
                                             (4096, 3072, 1536, True), (300, 1024, 5120, False)])
def test_nvfp4_graph_replay_matches_separate_calls(M, N, K, per_token):
    A, W, bias = _inputs(M, N, K, seed=M + N)
    layer = api.NVFP4Linear(W, bias, per_token=per_token)
    refs = [_separate(layer, a) for a in A]
    assert not torch.equal(refs[0], refs[1])

    x = A[0].clone()
    xq = layer.quantize_input(x)
    D = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        api.nvfp4_quantize(x, None if per_token else layer.gs_x, per_row=per_token, out=xq)
        api.nvfp4_gemm(xq, layer.weight, layer.alpha, xq.row_inv_gs if per_token else None, layer.bias, out=D)
    for i in (1, 2, 0, 1):
        x.copy_(A[i])
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(D, refs[i]), f"replay with input {i}"
    assert api.device_status() == 0


def test_back_to_back_launches_match_separate_calls():
    """quantize, GEMM, quantize, GEMM ... on one stream without synchronising."""
    M, N, K = 2048, 2048, 1536
    A, W, bias = _inputs(M, N, K, seed=7)
    layer = api.NVFP4Linear(W, bias)
    refs = [_separate(layer, a) for a in A]
    outs = [layer(a) for a in A for _ in range(2)]
    torch.cuda.synchronize()
    for j, y in enumerate(outs):
        assert torch.equal(y, refs[j // 2])
    assert api.device_status() == 0


def test_mxfp8_graph_replay_matches_separate_calls():
    M, N, K = 640, 1024, 2048
    A, W, bias = _inputs(M, N, K, seed=11)
    layer = api.MXFP8Linear(W, bias)
    refs = []
    for a in A:
        xq = api.mxfp8_quantize(a)
        torch.cuda.synchronize()
        refs.append(api.mxfp8_gemm(xq, layer.weight, None, layer.bias))
        torch.cuda.synchronize()
    x = A[0].clone()
    xq = api.mxfp8_quantize(x)
    D = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        api.mxfp8_quantize(x, out=xq)
        api.mxfp8_gemm(xq, layer.weight, None, layer.bias, out=D)
    for i in (2, 1, 0):
        x.copy_(A[i])
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(D, refs[i]), f"replay with input {i}"
    assert np.isfinite(D.float().cpu().numpy()).all()
    assert api.device_status() == 0
