"""fp64 oracle of the block epilogue and prologue around the mixer (test infrastructure).

Only ``tests/`` may import it. Source: "Gated DeltaNet-2: Decoupling Erase and
Write in Linear Attention" (graygoo.forestry.md note), sec. 3, block data-flow
paragraph: the mixer output is rescaled by an RMSNorm combined with a SiLU
gate (a GLU-style output gate). The note gives neither the epsilon nor where
the gate's projection comes from; the reading taken here (and by the CUDA
path) is the usual one:

    y[t, j] = o[t, j] / sqrt(mean_j' o[t, j']^2 + eps) * weight[j] * silu(g[t, j])
    silu(x) = x / (1 + exp(-x))

with the mean over the d_v channels of one head and one token, weight a
learned vector of d_v entries, and g a second projection of the block's input
with the shape of o. Either factor may be absent (weight None: no
normalisation; g None: no gate).
"""
from __future__ import annotations

import numpy as np


def silu(x):
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def output_norm_gate(o, g=None, weight=None, eps=1e-6):
    """y = RMSNorm(o) * weight (*) silu(g) over the last axis; fp64."""
    y = np.asarray(o, dtype=np.float64)
    if weight is not None:
        ms = np.mean(y * y, axis=-1, keepdims=True)
        y = y / np.sqrt(ms + eps) * np.asarray(weight, dtype=np.float64)
    if g is not None:
        y = y * silu(g)
    return y


# ---------------------------------------------------------------- block prologue
# Same note, sec. 3, block data-flow paragraph: query and key share a
# linear -> conv -> SiLU -> L2-norm path (the convolution adds local context), the value
# takes linear -> conv -> SiLU without the norm, and three separate branches give the
# per-channel decay alpha, erase gate b and write gate w. The note names neither the
# convolution's width nor the gate activations; the readings taken here (and by the CUDA
# path) are:
#   * the convolution is causal and depthwise over time, with the tap layout of a
#     depthwise Conv1d weight [C, 1, W] left-padded by W - 1: tap i multiplies the input
#     W - 1 - i tokens back, so the last tap is the current token; a state holds the
#     W - 1 inputs before the first token (oldest first), zeros when absent;
#   * L2 norm over the key channels of one head: x / sqrt(sum x^2 + eps);
#   * log alpha = -softplus(a) (alpha = sigmoid(-a) in (0, 1)), b = sigmoid(.), w = sigmoid(.):
#     the laws of the benchmark configurations.


def causal_conv(x, weight, state=None):
    """Depthwise causal convolution along the time axis (-2) of x [..., T, C].

    weight [C, W]: y[t, c] = sum_i weight[c, i] x[t - (W - 1) + i, c], with x at negative
    times taken from state [..., W - 1, C] (oldest first) or zero.
    """
    x = np.asarray(x, dtype=np.float64)
    wgt = np.asarray(weight, dtype=np.float64)
    W = wgt.shape[1]
    T = x.shape[-2]
    lead = x.shape[:-2]
    pad = np.zeros(lead + (W - 1, x.shape[-1])) if state is None else np.asarray(state, dtype=np.float64)
    xp = np.concatenate([pad, x], axis=-2)  # time index t of x sits at t + W - 1
    y = np.zeros_like(x)
    for i in range(W):
        y += wgt[:, i] * xp[..., i:i + T, :]
    return y


def conv_state_after(x, W, state=None):
    """The W - 1 inputs a continuing call needs: the last W - 1 of [state; x]."""
    x = np.asarray(x, dtype=np.float64)
    pad = np.zeros(x.shape[:-2] + (W - 1, x.shape[-1])) if state is None else np.asarray(state, dtype=np.float64)
    return np.concatenate([pad, x], axis=-2)[..., x.shape[-2]:, :]


def l2_normalize(x, eps=1e-6):
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def sigmoid(x):
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * (1.0 + np.tanh(0.5 * x))


def neg_softplus(x):
    """log alpha = -softplus(x) = -log(1 + e^x), without overflow."""
    x = np.asarray(x, dtype=np.float64)
    return -(np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x))))


def short_conv_silu(x, weight, state=None, l2norm=False, eps=1e-6, heads=1, cu_seqlens=None, states=None):
    """conv -> SiLU (-> L2 norm per head) of x [B, T, H * d] (or packed [1, T, H * d]).

    With cu_seqlens, each packed sequence i convolves on its own from states[i] ([W - 1, C]
    or zeros). Returns (y, state_after) with state_after [B or N, W - 1, C].
    """
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(weight).shape[1]
    if cu_seqlens is None:
        y = silu(causal_conv(x, weight, state))
        st = conv_state_after(x, W, state)
    else:
        y = np.zeros_like(x)
        st = []
        for i in range(len(cu_seqlens) - 1):
            s, e = int(cu_seqlens[i]), int(cu_seqlens[i + 1])
            si = None if states is None else states[i][None]
            y[:, s:e] = silu(causal_conv(x[:, s:e], weight, si))
            st.append(conv_state_after(x[:, s:e], W, si)[0])
        st = np.stack(st)
    if l2norm:
        sh = y.shape
        y = l2_normalize(y.reshape(sh[:-1] + (heads, sh[-1] // heads)), eps).reshape(sh)
    return y, st
