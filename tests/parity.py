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


def epilogue_err(y, y_ref, o_ref, g=None, weight=None, eps=1e-6) -> float:
    """Error of the normalised, gated output y = o / r * weight (.) silu(g), expressed as the
    mixer error (relative to max|o_ref|) that it implies.

    The per-token normalisation divides by r_t = sqrt(mean_j o_tj^2 + eps), which is small
    for tokens whose output nearly cancels, so a mixer error that passes the max-relative
    bound can move such a token's y by much more. To first order a mixer error do moves y
    by dy_j = w_j s_j (do_j / r - o_j dr / r^2) with s = silu(g) and
    |dr| <= rms(do) <= max|do|, hence |dy_tj| <= scale_t max|do| with
    scale_t = max_j |w_j s_tj| (1 + |o_tj| / r_t) / r_t (without a norm: max_j |s_tj|).
    The statistic is max_tj |y - y_ref| / (scale_t max|o_ref|): at most the mixer's own
    max-relative error, plus 2^-9 for the bf16 rounding of y.
    """
    from oracle.block import silu

    yg = y.detach().to("cpu", torch.float64).numpy() if isinstance(y, torch.Tensor) else np.asarray(y)
    o = np.asarray(o_ref, dtype=np.float64)
    assert yg.shape == o.shape == np.shape(y_ref)
    if o.size == 0:
        return 0.0
    if not np.all(np.isfinite(yg)):
        return float("inf")
    s = np.ones_like(o) if g is None else silu(g)
    ws = s * (1.0 if weight is None else np.asarray(weight, dtype=np.float64))
    if weight is not None:
        r = np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
        scale = np.max(np.abs(ws) * (1.0 + np.abs(o) / r), axis=-1, keepdims=True) / r
    else:
        scale = np.max(np.abs(ws), axis=-1, keepdims=True)
    denom = scale * float(np.max(np.abs(o)))
    diff = np.abs(yg - np.asarray(y_ref, dtype=np.float64))
    return float(np.max(np.where(denom > 0, diff / np.where(denom > 0, denom, 1.0), diff)))


def assert_epilogue_close(y, y_ref, o_ref, g, weight, eps, tol, what):
    e = epilogue_err(y, y_ref, o_ref, g, weight, eps)
    assert e <= tol, f"{what}: implied mixer error {e:.3e} > {tol:.1e}"
    return e
