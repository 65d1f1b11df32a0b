"""Seeded synthetic inputs for the block-scaled linear-layer workloads.

This module only draws data: it holds none of the quantization or GEMM
arithmetic, imports nothing else from this package, and serves both the CUDA
path (tests, benchmark) and the CPU oracle (tests, CPU baseline).

Every tensor is drawn on the host with ``numpy.random.default_rng(seed)`` in
float32 and rounded to bf16 (nearest-even) -- the same bytes on every machine.
``N(0, s)`` means a normal with standard deviation ``s``.  Outliers are a
per-entry Bernoulli(0.001) mask whose entries are multiplied by 50.  The GELU
that shapes the second FFN input is the tanh form, evaluated in float32.

Workloads (shapes of diffusion-transformer linears; the pages name the Wan-2.1
attention and FFN projections as the quantized layers in
hao-ai-lab-FastVideo nvfp4_qat_config.py, ``DEFAULT_FP4_LAYERS``):

  tiny      A [128, 256] ~N(0,1); W [256, 256] ~N(0, 0.02); no bias; seed 0
  wan13     A [32760, 1536] ~N(0,1) + outliers; W [1536, 1536] ~N(0, 1/sqrt(1536));
            bias [1536] ~N(0, 0.01); seed 1
  wan14_in  A [32760, 5120] ~N(0,1); W [13824, 5120] ~N(0, 1/sqrt(5120)); seed 2
  wan14_out A = bf16(gelu_tanh(N(0,1))) [32760, 13824]; W [5120, 13824] ~N(0, 1/sqrt(13824));
            seed 3 (the GELU of an fc_in-like output, drawn independently)
  skinny    A [M, 5120] ~N(0,1), M in {1, 16, 128, 1024, 4096}; W [13824, 5120] ~N(0, 0.02);
            seed 4
  skinny_out A [M, 13824] ~N(0,1); W [5120, 13824] ~N(0, 0.02) (the fc_out shape at
            decode-sized M); seed 7
  mxfp8     A [32760, 5120] ~N(0,1) + outliers; W [5120, 5120] ~N(0, 1/sqrt(5120)); seed 5
  weights   the 240 weights of 40 DiT blocks (q, k, v, out 5120x5120; fc_in 13824x5120;
            fc_out 5120x13824) ~N(0, 0.02), drawn on the device by ``device_weight``
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# 32760 tokens = 21 latent frames x 30 x 52 patches of a Wan-2.1 480p clip.
WAN_TOKENS = 32760
SKINNY_M = (1, 16, 128, 1024, 4096)
DIT_BLOCKS = 40
DIT_HIDDEN = 5120
DIT_FFN = 13824


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Nearest-even bf16 bit patterns (uint16) of finite float32 data."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(rng: np.random.Generator, shape, std: float = 1.0, outliers: bool = False) -> np.ndarray:
    x = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    if outliers:
        mask = rng.random(shape, dtype=np.float32) < np.float32(0.001)
        x[mask] *= np.float32(50.0)
    return f32_to_bf16_bits(x)


def gelu_tanh_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    x = rng.standard_normal(shape, dtype=np.float32)
    c = np.float32(math.sqrt(2.0 / math.pi))
    y = np.float32(0.5) * x * (np.float32(1.0) + np.tanh(c * (x + np.float32(0.044715) * x * x * x)))
    return f32_to_bf16_bits(y.astype(np.float32))


@dataclass
class Linear:
    """One linear layer's inputs as bf16 bit patterns: A [M, K], W [N, K], bias [N] or None."""
    name: str
    A: np.ndarray
    W: np.ndarray
    bias: np.ndarray | None = None
    per_token: bool = False
    meta: dict = field(default_factory=dict)

    @property
    def M(self) -> int:
        return self.A.shape[0]

    @property
    def N(self) -> int:
        return self.W.shape[0]

    @property
    def K(self) -> int:
        return self.A.shape[1]

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K


def tiny(M: int = 128, N: int = 256, K: int = 256, seed: int = 0) -> Linear:
    rng = np.random.default_rng(seed)
    return Linear("tiny", normal_bf16(rng, (M, K)), normal_bf16(rng, (N, K), 0.02))


def wan13(M: int = WAN_TOKENS, seed: int = 1) -> Linear:
    rng = np.random.default_rng(seed)
    K = N = 1536
    A = normal_bf16(rng, (M, K), outliers=True)
    W = normal_bf16(rng, (N, K), 1.0 / math.sqrt(K))
    bias = normal_bf16(rng, (N,), 0.01)
    return Linear("wan13", A, W, bias)


def wan14_in(M: int = WAN_TOKENS, seed: int = 2) -> Linear:
    rng = np.random.default_rng(seed)
    A = normal_bf16(rng, (M, DIT_HIDDEN))
    W = normal_bf16(rng, (DIT_FFN, DIT_HIDDEN), 1.0 / math.sqrt(DIT_HIDDEN))
    return Linear("wan14_in", A, W)


def wan14_out(M: int = WAN_TOKENS, seed: int = 3) -> Linear:
    rng = np.random.default_rng(seed)
    A = gelu_tanh_bf16(rng, (M, DIT_FFN))
    W = normal_bf16(rng, (DIT_HIDDEN, DIT_FFN), 1.0 / math.sqrt(DIT_FFN))
    return Linear("wan14_out", A, W)


def skinny(M: int, seed: int = 4) -> Linear:
    """Per-token-scaled activations against one fc_in-shaped weight."""
    rng = np.random.default_rng(seed)
    W = normal_bf16(rng, (DIT_FFN, DIT_HIDDEN), 0.02)
    A = normal_bf16(np.random.default_rng([seed, M]), (M, DIT_HIDDEN))
    return Linear(f"skinny_m{M}", A, W, per_token=True)


def skinny_out(M: int, seed: int = 7) -> Linear:
    """Per-token-scaled activations against one fc_out-shaped weight [5120, 13824]
    (few weight panels, long K)."""
    rng = np.random.default_rng(seed)
    W = normal_bf16(rng, (DIT_HIDDEN, DIT_FFN), 0.02)
    A = normal_bf16(np.random.default_rng([seed, M]), (M, DIT_FFN))
    return Linear(f"skinny_out_m{M}", A, W, per_token=True)


def mxfp8(M: int = WAN_TOKENS, seed: int = 5) -> Linear:
    rng = np.random.default_rng(seed)
    A = normal_bf16(rng, (M, DIT_HIDDEN), outliers=True)
    W = normal_bf16(rng, (DIT_HIDDEN, DIT_HIDDEN), 1.0 / math.sqrt(DIT_HIDDEN))
    return Linear("mxfp8", A, W)


def dit_weight_shapes(blocks: int = DIT_BLOCKS):
    """(block, name, N, K) of every linear in the synthetic DiT stack."""
    out = []
    for b in range(blocks):
        for name in ("to_q", "to_k", "to_v", "to_out"):
            out.append((b, name, DIT_HIDDEN, DIT_HIDDEN))
        out.append((b, "ffn.fc_in", DIT_FFN, DIT_HIDDEN))
        out.append((b, "ffn.fc_out", DIT_HIDDEN, DIT_FFN))
    return out


def device_weight(block: int, index: int, N: int, K: int, device, seed: int = 6):
    """One N(0, 0.02) bf16 weight drawn on ``device`` from a seeded torch generator.

    Used for the 9.86 G-element load-time sweep, too large to draw on the host.
    """
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(seed * 1_000_003 + block * 16 + index)
    return (torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * 0.02).to(torch.bfloat16)
