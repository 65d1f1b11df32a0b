"""Helpers for the GPU parity tests: host <-> device copies and the GEMM
tolerance, shared by tests/test_gpu_*.py."""
import numpy as np
import torch

import oracle

DEV = torch.device("cuda:0")


def up_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).view(torch.bfloat16).to(DEV)


def up(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def down(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return oracle.bf16_bits_to_f64(bits)


def ulp_bf16(y: np.ndarray) -> np.ndarray:
    a = np.maximum(np.abs(y), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7)


def gemm_tolerance(ref: np.ndarray, bound: np.ndarray, out_bf16: bool) -> np.ndarray:
    """Allowed |D_gpu - y| per element.

    fp32 output: 1e-3 * |alpha * row_scale| * sum_k |a_k b_k| (the accumulation
    bound).  bf16 output: that plus one bf16 ulp of y for the final rounding.
    """
    tol = 1e-3 * bound
    if out_bf16:
        tol = tol + ulp_bf16(ref)
    return tol


def assert_gemm_close(d_gpu: torch.Tensor, ref: np.ndarray, bound: np.ndarray, what: str = "") -> None:
    out_bf16 = d_gpu.dtype == torch.bfloat16
    got = bf16_to_f64(down(d_gpu)) if out_bf16 else down(d_gpu).astype(np.float64)
    assert got.shape == ref.shape
    tol = gemm_tolerance(ref, bound, out_bf16)
    err = np.abs(got - ref)
    bad = ~(err <= tol)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        detail = [(tuple(int(v) for v in i), float(got[tuple(i)]), float(ref[tuple(i)]), float(tol[tuple(i)]))
                  for i in idx]
        raise AssertionError(f"{what}: {int(bad.sum())}/{bad.size} outputs out of tolerance, e.g. {detail}")
    if out_bf16:
        # spec form: after rounding, within one bf16 ulp of bf16(y) wherever
        # the accumulation bound is below half an ulp
        near = 1e-3 * bound < 0.5 * ulp_bf16(ref)
        rb = bf16_to_f64(oracle.bf16_round(ref))
        assert np.all(np.abs(got - rb)[near] <= ulp_bf16(rb)[near]), what


def band_rows(M: int, bands) -> np.ndarray:
    """Row indices of the chosen 128-row scale bands, clipped to M."""
    rows = [np.arange(b * 128, min(M, b * 128 + 128)) for b in bands]
    return np.concatenate(rows) if rows else np.zeros(0, np.int64)


def sample_bands(M: int, n: int, seed: int = 0) -> list:
    """n random 128-row bands plus the first and the last (ragged) band."""
    nb = -(-M // 128)
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(nb, size=min(n, nb), replace=False).tolist()) | {0, nb - 1}
    return sorted(pick)
