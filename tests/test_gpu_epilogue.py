"""GPU parity of the block's output epilogue (RMSNorm with a SiLU output gate) fused
into the forward's output store, against the fp64 oracle: the oracle's forward,
then its epilogue (Gated DeltaNet-2 note, sec. 3, block data-flow paragraph).

The normalisation divides each token by its own rms, which amplifies the mixer's
tolerated error on tokens whose output nearly cancels; the full-path checks
therefore carry the mixer's bound through the normalisation (parity.epilogue_err),
and a well-conditioned case (every token's output of similar size) holds the
epilogue to the plain max-relative bound with weights and eps that expose a wrong
weight, eps or reduction."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from oracle.block import output_norm_gate
from gated_delta_rule_wy_b200 import GDR2Error, gdr2_forward, gdr2_forward_varlen, gdr2_sync_status
from gated_delta_rule_wy_b200 import inputs as I
from parity import TOL, assert_close, assert_epilogue_close, head_slice

pytestmark = pytest.mark.gpu

PARTS = {"norm_and_gate": (True, True), "norm_only": (True, False), "gate_only": (False, True)}


def _ref(n, g, wt, eps):
    o_ref, S_ref = oracle.forward(n["q"], n["k"], n["v"], n["log_alpha"], n["b"], n["w"], S0=n["S0"])
    return output_norm_gate(o_ref, g, wt, eps), o_ref, S_ref


@pytest.mark.parametrize("part", list(PARTS))
@pytest.mark.parametrize("T, la_shift", [(200, 0.0), (64, 0.0), (130, -30.0)])  # ragged, one chunk, exact path
def test_dense_epilogue_matches_the_oracle(part, T, la_shift):
    use_n, use_g = PARTS[part]
    x = I.make_forward_inputs(B=2, H=3, T=T, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=91,
                              with_S0=True)
    x = dataclasses.replace(x, log_alpha=x.log_alpha + la_shift)
    g, wt = I.make_epilogue_inputs((2, T, 3, 128), 128, seed=92)
    d = x.to("cuda")
    eps = 1e-6
    o, S_T, _ = gdr2_forward(d.q, d.k, d.v, d.log_alpha, d.b, d.w, d.S0,
                             out_gate=g.cuda() if use_g else None, norm_weight=wt.cuda() if use_n else None,
                             norm_eps=eps)
    gdr2_sync_status()
    n = x.as_numpy64()
    gn, wn = g.double().numpy() if use_g else None, wt.double().numpy() if use_n else None
    y_ref, o_ref, S_ref = _ref(n, gn, wn, eps)
    assert_epilogue_close(o, y_ref, o_ref, gn, wn, eps, TOL[torch.bfloat16], f"{part} T={T}: y")
    assert_close(S_T, S_ref, TOL[torch.bfloat16], f"{part} T={T}: S_T")


@pytest.mark.parametrize("eps", [1e-6, 1e-2])
@pytest.mark.parametrize("T", [200, 64])
def test_well_conditioned_epilogue_plain_bound(eps, T):
    """k = 0 and no decay: o_t = S0^T q_t, every token's output of rms about 0.1. The plain
    max-relative bound then applies to y; weights ~ N(0, 1) and eps = 1e-2 (comparable to
    the mean square) make a wrong weight, eps or reduction width fail it."""
    x = I.make_forward_inputs(B=2, H=3, T=T, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=101,
                              with_S0=True)
    x = dataclasses.replace(x, k=torch.zeros_like(x.k), log_alpha=torch.zeros_like(x.log_alpha))
    g, _ = I.make_epilogue_inputs((2, T, 3, 128), 128, seed=102)
    wt = torch.randn(128, generator=torch.Generator().manual_seed(103))
    d = x.to("cuda")
    y, _, _ = gdr2_forward(d.q, d.k, d.v, d.log_alpha, d.b, d.w, d.S0, out_gate=g.cuda(), norm_weight=wt.cuda(),
                           norm_eps=eps)
    gdr2_sync_status()
    y_ref, _, _ = _ref(x.as_numpy64(), g.double().numpy(), wt.double().numpy(), eps)
    assert_close(y, y_ref, TOL[torch.bfloat16], f"well-conditioned eps={eps} T={T}: y")


def test_epilogue_leaves_the_states_alone():
    """S_T and the saved chunk states are the recurrence's: bit-equal with and without."""
    x = I.make_forward_inputs(B=1, H=4, T=300, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=93,
                              with_S0=True)
    g, wt = I.make_epilogue_inputs((1, 300, 4, 128), 128, seed=94)
    d = x.to("cuda")
    _, S_a, sv_a = gdr2_forward(d.q, d.k, d.v, d.log_alpha, d.b, d.w, d.S0, save_states=True)
    _, S_b, sv_b = gdr2_forward(d.q, d.k, d.v, d.log_alpha, d.b, d.w, d.S0, save_states=True,
                                out_gate=g.cuda(), norm_weight=wt.cuda())
    gdr2_sync_status()
    assert torch.equal(S_a, S_b) and torch.equal(sv_a, sv_b)


def test_unit_norm_rows_and_saturated_gates():
    """weight = 1 and eps = 0: every token's output has rms 1 (to bf16 rounding; with eps > 0
    a token of mean square m would have sqrt(m / (m + eps))); gates at +-40 pass o through
    scaled by 40 or shut it (silu(-40) ~ -1.7e-16)."""
    B, T, H = 1, 192, 2
    x = I.make_forward_inputs(B=B, H=H, T=T, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=95,
                              with_S0=True)
    d = x.to("cuda")
    one = torch.ones(128, device="cuda")
    y, _, _ = gdr2_forward(d.q, d.k, d.v, d.log_alpha, d.b, d.w, d.S0, norm_weight=one, norm_eps=0.0)
    gdr2_sync_status()
    rms = y.float().pow(2).mean(-1).sqrt()
    assert torch.allclose(rms, torch.ones_like(rms), atol=4e-3), float((rms - 1).abs().max())
    sign = torch.where(torch.arange(T) % 2 == 0, 40.0, -40.0)[None, :, None, None]
    g = (sign * torch.ones(B, T, H, 128)).to(torch.bfloat16).cuda()
    z, _, _ = gdr2_forward(d.q, d.k, d.v, d.log_alpha, d.b, d.w, d.S0, out_gate=g, norm_weight=one, norm_eps=0.0)
    gdr2_sync_status()
    assert z[:, 1::2].float().abs().max().item() < 1e-12
    assert torch.allclose(z[:, 0::2].float(), 40.0 * y[:, 0::2].float(), rtol=8e-3, atol=0)


@pytest.mark.parametrize("part", list(PARTS))
def test_packed_sequences_with_the_epilogue(part):
    use_n, use_g = PARTS[part]
    lens = [0, 70, 1, 128, 33, 64]
    T, H = sum(lens), 2
    x = I.make_forward_inputs(B=1, H=H, T=T, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=96)
    S0 = torch.randn((len(lens), H, 128, 128), generator=torch.Generator().manual_seed(97)) * 0.1
    cu = np.concatenate([[0], np.cumsum(lens)])
    g, wt = I.make_epilogue_inputs((T, H, 128), 128, seed=98)
    d = x.to("cuda")
    o, S_T, _ = gdr2_forward_varlen(d.q, d.k, d.v, d.log_alpha, d.b, d.w,
                                    torch.tensor(cu, dtype=torch.int32, device="cuda"), S0.cuda(),
                                    out_gate=g.cuda() if use_g else None, norm_weight=wt.cuda() if use_n else None)
    gdr2_sync_status()
    n = x.as_numpy64()
    gn, wn = g.double().numpy(), wt.double().numpy()
    for i in range(len(lens)):
        s, e = int(cu[i]), int(cu[i + 1])
        if e == s:
            assert torch.equal(S_T[i].cpu(), S0[i])
            continue
        args = [n[f][:, s:e] for f in ("q", "k", "v", "log_alpha", "b", "w")]
        o_ref, S_ref = oracle.forward(*args, S0=S0[i:i + 1].double().numpy())
        gi, wi = gn[None, s:e] if use_g else None, wn if use_n else None
        y_ref = output_norm_gate(o_ref, gi, wi, 1e-6)
        assert_epilogue_close(o[s:e][None], y_ref, o_ref, gi, wi, 1e-6, TOL[torch.bfloat16],
                              f"{part} seq {i} (len {e - s}): y")
        assert_close(S_T[i:i + 1], S_ref, TOL[torch.bfloat16], f"{part} seq {i}: S_T")


def test_epilogue_needs_the_tensor_core_path():
    x = I.make_forward_inputs(B=1, H=1, T=64, dk=64, dv=64, dtype=torch.float32, seed=99)
    d = x.to("cuda")
    with pytest.raises(GDR2Error, match="UNSUPPORTED"):
        gdr2_forward(d.q, d.k, d.v, d.log_alpha, d.b, d.w, None, norm_weight=torch.ones(64, device="cuda"))


@pytest.mark.slow
def test_full_size_1p3b_layer_with_epilogue_sampled_heads():
    """B=4 H=16 T=4096 d=128 bf16 with norm and gate; oracle on sampled heads."""
    x = I.make_forward_inputs(**I.FWD_1P3B_BF16)
    g, wt = I.make_epilogue_inputs((4, 4096, 16, 128), 128, seed=100)
    d = x.to("cuda")
    y, S_T, _ = gdr2_forward(d.q, d.k, d.v, d.log_alpha, d.b, d.w, d.S0, out_gate=g.cuda(), norm_weight=wt.cuda())
    gdr2_sync_status()
    assert torch.isfinite(y.float()).all()
    n = x.as_numpy64()
    gn, wn = g.double().numpy(), wt.double().numpy()
    for (b, h) in [(0, 3), (2, 11)]:
        args = [head_slice(n[f], b, h) for f in ("q", "k", "v", "log_alpha", "b", "w")]
        o_ref, S_ref = oracle.forward(*args, S0=head_slice(n["S0"], b, h, token_major=False))
        gi = head_slice(gn, b, h)
        y_ref = output_norm_gate(o_ref, gi, wn, 1e-6)
        assert_epilogue_close(y[b:b + 1, :, h:h + 1], y_ref, o_ref, gi, wn, 1e-6, TOL[torch.bfloat16],
                              f"y[b={b},h={h}]")
        assert_close(S_T[b:b + 1, h:h + 1], S_ref, TOL[torch.bfloat16], f"S_T[b={b},h={h}]")


def test_one_token_with_the_epilogue():
    """T = 1: one partial chunk, its gate tile clipped to one row."""
    x = I.make_forward_inputs(B=3, H=2, T=1, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=104,
                              with_S0=True)
    g, _ = I.make_epilogue_inputs((3, 1, 2, 128), 128, seed=105)
    wt = torch.randn(128, generator=torch.Generator().manual_seed(106))
    d = x.to("cuda")
    y, _, _ = gdr2_forward(d.q, d.k, d.v, d.log_alpha, d.b, d.w, d.S0, out_gate=g.cuda(), norm_weight=wt.cuda(),
                           norm_eps=1e-2)
    gdr2_sync_status()
    n = x.as_numpy64()
    o_ref, _ = oracle.forward(n["q"], n["k"], n["v"], n["log_alpha"], n["b"], n["w"], S0=n["S0"])
    y_ref = output_norm_gate(o_ref, g.double().numpy(), wt.double().numpy(), 1e-2)
    assert_epilogue_close(y, y_ref, o_ref, g.double().numpy(), wt.double().numpy(), 1e-2, TOL[torch.bfloat16], "T=1 y")


def test_packed_scalar_gates_with_the_epilogue():
    """Packed sequences, b = w = beta per token-head and the output norm and gate, all in one
    gdr2_forward_ex call, against the oracle sequence by sequence."""
    lens = [50, 0, 129, 7]
    T, H = sum(lens), 2
    x = I.make_forward_inputs(B=1, H=H, T=T, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=107)
    beta = torch.sigmoid(torch.randn((T, H), generator=torch.Generator().manual_seed(108))).to(torch.bfloat16)
    g, wt = I.make_epilogue_inputs((T, H, 128), 128, seed=109)
    cu = np.concatenate([[0], np.cumsum(lens)])
    d = x.to("cuda")
    y, S_T, _ = gdr2_forward_varlen(d.q, d.k, d.v, d.log_alpha, beta.cuda(), beta.cuda(),
                                    torch.tensor(cu, dtype=torch.int32, device="cuda"), out_gate=g.cuda(),
                                    norm_weight=wt.cuda())
    gdr2_sync_status()
    n = x.as_numpy64()
    bv = np.repeat(beta.double().numpy()[None, ..., None], 128, axis=-1)
    gn, wn = g.double().numpy(), wt.double().numpy()
    for i in range(len(lens)):
        s, e = int(cu[i]), int(cu[i + 1])
        if e == s:
            assert torch.count_nonzero(S_T[i]) == 0
            continue
        o_ref, S_ref = oracle.forward(n["q"][:, s:e], n["k"][:, s:e], n["v"][:, s:e], n["log_alpha"][:, s:e],
                                      bv[:, s:e], bv[:, s:e])
        y_ref = output_norm_gate(o_ref, gn[None, s:e], wn, 1e-6)
        assert_epilogue_close(y[s:e][None], y_ref, o_ref, gn[None, s:e], wn, 1e-6, TOL[torch.bfloat16], f"seq {i}")
        assert_close(S_T[i:i + 1], S_ref, TOL[torch.bfloat16], f"seq {i} S_T")
