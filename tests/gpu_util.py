"""Helpers shared by the GPU parity tests (conversions and comparisons)."""
from __future__ import annotations

import numpy as np
import torch


def to_np(t: torch.Tensor) -> np.ndarray:
    """Any CUDA tensor -> float64 NumPy array (bf16 and fp32 values are exact)."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def to_bf16(x: np.ndarray) -> torch.Tensor:
    """float64 array of bf16-representable values -> bf16 CUDA tensor (exact)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to("cuda").to(torch.bfloat16)


def to_f32(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to("cuda")


def rel_fro(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.linalg.norm(ref))
    return float(np.linalg.norm(x - ref)) / (den if den > 0 else 1.0)


def bf16_ulp(x) -> np.ndarray:
    """Spacing of bf16 values at |x| (2^(e-7)), with the subnormal floor."""
    ax = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


def bf16_agreement(gpu, ref):
    """(mismatch fraction, max |gpu-ref| in bf16 ulps of the larger value)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = np.abs(gpu - ref)
    mism = float(np.mean(diff > 0)) if diff.size else 0.0
    if not diff.size:
        return 0.0, 0.0
    ulps = diff / bf16_ulp(np.maximum(np.abs(gpu), np.abs(ref)))
    return mism, float(ulps.max())


def bf16_close(gpu, ref, acc_bound):
    """Worst ratio |gpu - ref| / (1 bf16 ulp + acc_bound), elementwise.

    acc_bound is an elementwise bound on the difference between the GPU's
    fp32-accumulated value and the oracle's fp64 value before the final bf16
    rounding; the rounding itself can add one ulp.  A ratio <= 1 everywhere
    means every difference is explained by accumulation order alone.
    """
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if not gpu.size:
        return 0.0
    tol = bf16_ulp(np.maximum(np.abs(gpu), np.abs(ref))) + np.asarray(acc_bound, dtype=np.float64)
    return float(np.max(np.abs(gpu - ref) / tol))


def fp32_gemm_bound(a, b, k):
    """Error bound of an fp32-accumulated product a @ b of k terms: any order
    of k-1 roundings (2^-24 each; doubled for truncating adders)."""
    return 2.0 * k * 2.0 ** -24 * (np.abs(a) @ np.abs(b))
