"""Helpers shared by the GPU parity tests (the CUDA path against the fp64 oracle).

The statistic is max|gpu - ref| / max|ref| per output tensor; the bounds are
1e-4 for fp32 inputs and 2e-2 for bf16 inputs with an fp32 state.
"""
from __future__ import annotations

import numpy as np
import torch

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def rel_err(gpu, ref) -> float:
    g = gpu.detach().to("cpu", torch.float64).numpy() if isinstance(gpu, torch.Tensor) else np.asarray(gpu)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    if r.size == 0:
        return 0.0
    denom = float(np.max(np.abs(r)))
    err = float(np.max(np.abs(g - r)))
    if not np.all(np.isfinite(g)):
        return float("inf")
    return err / denom if denom > 0 else err


def assert_close(gpu, ref, tol, what):
    e = rel_err(gpu, ref)
    assert e <= tol, f"{what}: max|err|/max|ref| = {e:.3e} > {tol:.1e}"
    return e


def head_slice(x: np.ndarray | None, b: int, h: int, token_major: bool = True):
    """One (batch, head) of a [B, T, H, D] (token_major) or [B, H, ...] array, kept 4-D."""
    if x is None:
        return None
    if token_major:
        return np.ascontiguousarray(x[b:b + 1, :, h:h + 1])
    return np.ascontiguousarray(x[b:b + 1, h:h + 1])
