"""Load-time weight conversion in one kernel (nvfp4_quantize_weight, and
nvfp4_quantize_weights for many weights in one launch) on the GPU.

The entry fuses the weight path of sgl-project sglang nvfp4_online.py
(_quantize_weight_nvfp4: amax, gs = e4m3_max * 6 / amax, quantize) into one
cooperative launch with a grid barrier.  Its results must be bit-identical to
the three-launch sequence amax -> global scale -> nvfp4_quantize, and to the
oracle's amax, global scale and quantization."""
import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_05_b200 import _native as nat
from block_scaled_precision_05_b200 import api
from block_scaled_precision_05_b200 import workloads as wl
from tests._gpu import DEV, down, up_bf16

pytestmark = pytest.mark.gpu


def _bf16(rows, K, seed, std=0.02):
    rng = np.random.default_rng(seed)
    return wl.f32_to_bf16_bits((rng.standard_normal((rows, K)) * std).astype(np.float32))


def _three_launches(w, fmax):
    a = api.amax(w)
    gs, inv = api.nvfp4_global_scale(a, fmax)
    return api.nvfp4_quantize(w, gs), gs, inv, a


def _assert_same(fused, ref):
    (q1, g1, i1, a1), (q2, g2, i2, a2) = fused, ref
    assert torch.equal(q1.codes, q2.codes)
    assert torch.equal(q1.sf, q2.sf)
    for x, y in ((g1, g2), (i1, i2), (a1, a2)):
        assert torch.equal(x, y), (x, y)


SHAPES = [(1, 64), (7, 128), (130, 1536), (300, 5120), (1000, 13824), (5120, 5120), (13824, 5120), (333, 576)]


@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("fmax", [api.FP8_FP4_MAX, api.FP8_FP4_MAX_4OVER6])
def test_matches_three_launches(N, K, fmax):
    g = torch.Generator(device=DEV)
    g.manual_seed(N * 7 + K)
    w = (torch.randn((N, K), generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    fused = api.nvfp4_quantize_weight(w, fmax)
    ref = _three_launches(w, fmax)
    assert api.device_status() == 0
    _assert_same(fused, ref)


@pytest.mark.parametrize("N,K", [(1, 64), (130, 1536), (257, 640)])
def test_matches_oracle(N, K):
    W = _bf16(N, K, seed=N + K)
    q, gs, inv, a = api.nvfp4_quantize_weight(up_bf16(W))
    assert api.device_status() == 0
    a_ref = oracle.amax_bf16(W)
    g_ref = oracle.nvfp4_global_scale(a_ref)
    assert down(a)[0] == np.float32(a_ref)
    assert down(gs)[0] == g_ref and down(inv)[0] == np.float32(1.0) / g_ref
    codes, sf = oracle.nvfp4_quantize(W, g_ref)
    assert np.array_equal(down(q.codes), codes)
    assert np.array_equal(down(q.sf), sf)


def test_special_values_and_zero_weight():
    W = _bf16(200, 256, seed=5)
    W[3, 7] = 0x7F80   # +inf counts as the largest finite value
    W[9, 0] = 0x7FC1   # NaN counts as 0
    W[11, 1] = 0x0001  # subnormal
    w = up_bf16(W)
    _assert_same(api.nvfp4_quantize_weight(w), _three_launches(w, api.FP8_FP4_MAX))
    z = torch.zeros((130, 128), dtype=torch.bfloat16, device=DEV)
    q, gs, inv, a = api.nvfp4_quantize_weight(z)
    assert down(a)[0] == 0.0 and down(gs)[0] == 1.0 and down(inv)[0] == 1.0
    assert not q.codes.any() and not q.sf.any()
    assert api.device_status() == 0


def test_f16_weight():
    rng = np.random.default_rng(8)
    W = (rng.standard_normal((300, 1024)) * 30).astype(np.float16).view(np.uint16)
    W[0, 5] = 0xFC00  # -inf -> 65504
    w = torch.from_numpy(W.view(np.int16)).view(torch.float16).to(DEV)
    fused = api.nvfp4_quantize_weight(w)
    _assert_same(fused, _three_launches(w, api.FP8_FP4_MAX))
    g_ref = oracle.nvfp4_global_scale(oracle.amax_f16(W))
    assert down(fused[1])[0] == g_ref
    codes, sf = oracle.nvfp4_quantize(W, g_ref, fmt="f16")
    assert np.array_equal(down(fused[0].codes), codes) and np.array_equal(down(fused[0].sf), sf)


def test_strided_rows():
    g = torch.Generator(device=DEV)
    g.manual_seed(3)
    big = (torch.randn((700, 1600), generator=g, device=DEV) * 0.05).to(torch.bfloat16)
    w = big[:, :1536]
    assert w.stride(0) == 1600
    _assert_same(api.nvfp4_quantize_weight(w), _three_launches(w.contiguous(), api.FP8_FP4_MAX))


def test_consecutive_calls_reuse_the_workspace():
    """The grid barrier leaves its arrival count at 0: many calls in a row, on
    weights of different sizes, each match their own three-launch result."""
    g = torch.Generator(device=DEV)
    g.manual_seed(11)
    ws = [(torch.randn(s, generator=g, device=DEV) * sc).to(torch.bfloat16)
          for s, sc in (((512, 1024), 0.02), ((3, 64), 5.0), ((2048, 5120), 0.01), ((512, 1024), 0.3))]
    fused = [api.nvfp4_quantize_weight(w) for w in ws for _ in range(2)]
    torch.cuda.synchronize()
    for j, f in enumerate(fused):
        _assert_same(f, _three_launches(ws[j // 2], api.FP8_FP4_MAX))
    for ws_t in api._WEIGHT_WS.values():
        assert int(ws_t[:4].view(torch.int32)[0]) == 0
    assert api.device_status() == 0


def test_workspace_left_by_a_timed_out_call_is_fit_for_the_next():
    """A barrier wait that runs out leaves a non-zero arrival count (and stale
    block words) in the workspace.  Each call clears the barrier words on its
    stream before the launch, so a later call on that workspace is still
    correct.  The stale state is written by the host here; nothing waits."""
    g = torch.Generator(device=DEV)
    g.manual_seed(13)
    w = (torch.randn((3000, 5120), generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    w2 = (torch.randn((700, 1024), generator=g, device=DEV) * 2.0).to(torch.bfloat16)
    api.nvfp4_quantize_weight(w)  # sets up the per-device workspace
    torch.cuda.synchronize()
    ws = api._weight_workspace(DEV, nat.BSP_IN_BF16)
    words = ws.view(torch.int32)
    for stale in ((5, 3), (443, 0)):  # arrivals short of the grid, and one short of releasing
        words[0], words[1] = stale
        words[64:] = 0x7F7F0000  # block words of a larger amax than any here
        f1 = api.nvfp4_quantize_weight(w)
        words[0] = stale[0]
        f2 = api.nvfp4_quantize_weights([w2])[0]
        torch.cuda.synchronize()
        _assert_same(f1, _three_launches(w, api.FP8_FP4_MAX))
        _assert_same(f2, _three_launches(w2, api.FP8_FP4_MAX))
        assert int(words[0]) == 0
    assert api.device_status() == 0


def test_graph_replay():
    g = torch.Generator(device=DEV)
    g.manual_seed(12)
    w = (torch.randn((1024, 5120), generator=g, device=DEV) * 0.02).to(torch.bfloat16)
    q, gs, inv, a = api.nvfp4_quantize_weight(w)  # sets up the workspace outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        out = api.nvfp4_quantize_weight(w)
    for scale in (0.5, 3.0):
        w.mul_(scale)
        graph.replay()
        torch.cuda.synchronize()
        _assert_same(out, _three_launches(w, api.FP8_FP4_MAX))
    assert api.device_status() == 0


def test_layer_uses_it():
    W = _bf16(384, 1024, seed=21)
    layer = api.NVFP4Linear(up_bf16(W))
    g_ref = oracle.nvfp4_global_scale(oracle.amax_bf16(W))
    assert down(layer.gs_w)[0] == g_ref
    codes, sf = oracle.nvfp4_quantize(W, g_ref)
    assert np.array_equal(down(layer.weight.codes), codes) and np.array_equal(down(layer.weight.sf), sf)


def test_batch_matches_single_launches():
    """nvfp4_quantize_weights: one launch over mixed weights (ragged, L2-sized,
    larger than L2, a strided view, an all-zero weight) equals the
    single-weight entry on each."""
    g = torch.Generator(device=DEV)
    g.manual_seed(21)
    big = (torch.randn((700, 1600), generator=g, device=DEV) * 0.05).to(torch.bfloat16)
    weights = [(torch.randn(s, generator=g, device=DEV) * sc).to(torch.bfloat16)
               for s, sc in (((5120, 5120), 0.02), ((130, 1536), 1.0), ((7, 128), 3.0), ((13824, 5120), 0.02),
                             ((1000, 576), 0.5))]
    weights += [big[:, :1536], torch.zeros((129, 64), dtype=torch.bfloat16, device=DEV)]
    for fmax in (api.FP8_FP4_MAX, api.FP8_FP4_MAX_4OVER6):
        batch = api.nvfp4_quantize_weights(weights, fmax)
        for w, b in zip(weights, batch):
            _assert_same(b, api.nvfp4_quantize_weight(w, fmax))
    assert api.device_status() == 0


def test_batch_chunks_and_f16():
    """More weights than one launch takes (split into chunks), and fp16."""
    g = torch.Generator(device=DEV)
    g.manual_seed(22)
    n = 300
    weights = [(torch.randn((3 + i % 5, 64 * (1 + i % 3)), generator=g, device=DEV) * (0.1 + i)).to(torch.float16)
               for i in range(n)]
    batch = api.nvfp4_quantize_weights(weights)
    assert len(batch) == n
    for w, b in zip(weights, batch):
        _assert_same(b, api.nvfp4_quantize_weight(w))
    assert api.device_status() == 0


def test_batch_graph_replay():
    g = torch.Generator(device=DEV)
    g.manual_seed(23)
    weights = [(torch.randn(s, generator=g, device=DEV) * 0.02).to(torch.bfloat16) for s in ((1024, 5120), (256, 1536))]
    api.nvfp4_quantize_weights(weights)  # sets up the workspace outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        outs = api.nvfp4_quantize_weights(weights)
    for scale in (0.5, 7.0):
        for w in weights:
            w.mul_(scale)
        graph.replay()
        torch.cuda.synchronize()
        for w, b in zip(weights, outs):
            _assert_same(b, api.nvfp4_quantize_weight(w))
    assert api.device_status() == 0
