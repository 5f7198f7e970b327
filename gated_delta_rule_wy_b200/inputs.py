"""Seeded synthetic inputs for the GDR-2 token mixer.

This module only draws random numbers: it holds none of the mixer's
arithmetic, and both the CUDA path and the fp64 oracle take their inputs from
it. Tensors are drawn on the CPU with a ``torch.Generator`` in fp32, in a fixed
order, then cast to the input dtype; the oracle upcasts the cast values
exactly, so both sides see identical numbers.

Distributions follow the workloads of the Gated DeltaNet-2 note (1.3B-model
layers, H = 16 heads of d = 128; sec. 1 and sec. 4) and the block structure of
its sec. 3 (q and k leave the block prologue L2-normalised per token; the
decay, erase and write branches emit alpha in (0,1], b and w in [0,1]):

  q, k      ~ N(0,1), L2-normalised over the key dimension
  v         ~ N(0,1)
  log_alpha = -softplus(N(0,1) + shift)   (shift 0 for the fp32 case, 2 else)
  b, w      = sigmoid(N(0,1))
"""
from __future__ import annotations

import dataclasses

import torch

# Workloads, named by what they are.
FWD_SMALL_F32 = dict(B=1, H=1, T=256, dk=64, dv=64, dtype=torch.float32, decay_shift=0.0, seed=1000)
FWD_1P3B_BF16 = dict(B=4, H=16, T=4096, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=1001)
SWEEP_TOKENS = 65536
SWEEP_T = (2048, 4096, 8192, 16384, 32768)
DECODE_1P3B = dict(N=256, H=16, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=1003,
                   steps=512, state_std=0.02)
BWD_1P3B_BF16 = dict(B=2, H=16, T=4096, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=1004)


def sweep_config(T: int) -> dict:
    """Sequence-length sweep at a fixed 65,536 tokens per call (B = 65536 / T)."""
    if SWEEP_TOKENS % T:
        raise ValueError("T must divide 65536")
    return dict(B=SWEEP_TOKENS // T, H=16, T=T, dk=128, dv=128, dtype=torch.bfloat16,
                decay_shift=2.0, seed=1002)


@dataclasses.dataclass
class FwdInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    log_alpha: torch.Tensor
    b: torch.Tensor
    w: torch.Tensor
    S0: torch.Tensor | None

    def to(self, device) -> "FwdInputs":
        return FwdInputs(*(None if t is None else t.to(device) for t in dataclasses.astuple(self)))

    def as_numpy64(self) -> dict:
        out = {}
        for f in dataclasses.fields(self):
            t = getattr(self, f.name)
            out[f.name] = None if t is None else t.detach().to("cpu", torch.float64).numpy()
        return out


def _l2norm_rows(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def make_token_inputs(shape_k, shape_v, dtype, decay_shift, gen, normalise_qk=True):
    """Draw q, k, v, log_alpha, b, w with the distributions in the module docstring.

    Tensors are drawn on the generator's device (CPU, or CUDA for long decode runs).
    """
    dev = gen.device
    q = torch.randn(shape_k, generator=gen, device=dev)
    k = torch.randn(shape_k, generator=gen, device=dev)
    v = torch.randn(shape_v, generator=gen, device=dev)
    la = -torch.nn.functional.softplus(torch.randn(shape_k, generator=gen, device=dev) + decay_shift)
    b = torch.sigmoid(torch.randn(shape_k, generator=gen, device=dev))
    w = torch.sigmoid(torch.randn(shape_v, generator=gen, device=dev))
    if normalise_qk:
        q, k = _l2norm_rows(q), _l2norm_rows(k)
    return (q.to(dtype), k.to(dtype), v.to(dtype), la.to(torch.float32), b.to(dtype), w.to(dtype))


def make_forward_inputs(B, H, T, dk, dv, dtype=torch.float32, decay_shift=0.0, seed=0,
                        with_S0=False, S0_std=0.1, **_ignored) -> FwdInputs:
    """Inputs of one forward call in token-major [B, T, H, D] layout.

    S0 is None (zero initial state) unless ``with_S0``; then S0 ~ N(0, S0_std^2) fp32.
    """
    gen = torch.Generator().manual_seed(int(seed))
    q, k, v, la, b, w = make_token_inputs((B, T, H, dk), (B, T, H, dv), dtype, decay_shift, gen)
    S0 = torch.randn((B, H, dk, dv), generator=gen) * S0_std if with_S0 else None
    return FwdInputs(q, k, v, la, b, w, S0)


def make_decode_inputs(N, H, dk, dv, dtype=torch.bfloat16, decay_shift=2.0, seed=0, steps=1,
                       state_std=0.02, **_ignored):
    """Prior state S ~ N(0, state_std^2) fp32 [N, H, dk, dv] and ``steps`` tokens per sequence.

    Returns (S, tokens) with tokens a list of (q, k, v, log_alpha, b, w), each [N, H, D].
    """
    gen = torch.Generator().manual_seed(int(seed))
    S = torch.randn((N, H, dk, dv), generator=gen) * state_std
    toks = [make_token_inputs((N, H, dk), (N, H, dv), dtype, decay_shift, gen) for _ in range(steps)]
    return S, toks


def make_upstream_grad(B, T, H, dv, seed, dtype=torch.float32):
    """dO ~ N(0, 1) in the output layout [B, T, H, dv]."""
    gen = torch.Generator().manual_seed(int(seed) + 7919)
    return torch.randn((B, T, H, dv), generator=gen).to(dtype)


def make_epilogue_inputs(o_shape, dv, dtype=torch.bfloat16, seed=0, gate_scale=1.0):
    """Output-gate pre-activations and RMSNorm weight for the block epilogue.

    g ~ gate_scale * N(0, 1) in o's layout and dtype (a linear projection of the block
    input); weight = 1 + 0.1 N(0, 1) over the dv channels, fp32 (a learned norm weight
    near its initial value of one).
    """
    gen = torch.Generator().manual_seed(int(seed) + 104729)
    g = (torch.randn(tuple(o_shape), generator=gen) * gate_scale).to(dtype)
    weight = 1.0 + 0.1 * torch.randn((dv,), generator=gen)
    return g, weight


def make_conv_inputs(x_shape, W, dtype=torch.bfloat16, seed=0):
    """Short-convolution branch inputs: x ~ N(0, 1) (a projection's output) in x_shape
    ([N, T, H, d] or [T, H, d]); taps ~ U(-1/sqrt(W), 1/sqrt(W)) fp32 [H * d, W] (the usual
    initialisation of a depthwise convolution with W inputs per output); a state
    ~ N(0, 1) [N, W - 1, H, d] in dtype (N = x_shape[0])."""
    gen = torch.Generator().manual_seed(int(seed) + 130363)
    H, d = x_shape[-2], x_shape[-1]
    x = torch.randn(tuple(x_shape), generator=gen).to(dtype)
    wgt = (torch.rand((H * d, W), generator=gen) * 2 - 1) / W ** 0.5
    st = torch.randn((x_shape[0], W - 1, H, d), generator=gen).to(dtype)
    return x, wgt, st


def make_prologue_inputs(B, T, H, dk, dv, W, dtype=torch.bfloat16, seed=0, decay_shift=2.0):
    """Projection outputs for the whole block prologue: xq, xk [B, T, H, dk], xv [B, T, H, dv]
    ~ N(0, 1); convolution taps as in make_conv_inputs; decay pre-activation a ~ N(0, 1) +
    shift and gate pre-activations ~ N(0, 1), so that -softplus(a) and sigmoid give the
    mixer's input laws above."""
    gen = torch.Generator().manual_seed(int(seed) + 15485863)
    out = {}
    for name, dd in (("q", dk), ("k", dk), ("v", dv)):
        out["x" + name] = torch.randn((B, T, H, dd), generator=gen).to(dtype)
        out["conv_" + name] = (torch.rand((H * dd, W), generator=gen) * 2 - 1) / W ** 0.5
    out["a"] = (torch.randn((B, T, H, dk), generator=gen) + decay_shift).to(dtype)
    out["b"] = torch.randn((B, T, H, dk), generator=gen).to(dtype)
    out["w"] = torch.randn((B, T, H, dv), generator=gen).to(dtype)
    return out
