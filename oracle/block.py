"""fp64 oracle of the block epilogue around the mixer (test infrastructure).

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
