"""GPU parity of gdr2_decode_step against the fp64 oracle (needs a B200)."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_wy_b200 import gdr2_decode_step, gdr2_forward, gdr2_sync_status
from gated_delta_rule_wy_b200 import inputs as I
from parity import TOL, assert_close

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().to("cpu", torch.float64).numpy()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
def test_chained_steps(dtype, dk, dv):
    S, toks = I.make_decode_inputs(N=3, H=2, dk=dk, dv=dv, dtype=dtype, decay_shift=2.0, seed=7, steps=12,
                                   state_std=0.02)
    Sg = S.cuda()
    Sr = S.double().numpy()
    for i, tk in enumerate(toks):
        o = gdr2_decode_step(*(t.cuda() for t in tk), Sg)
        o_ref, Sr = oracle.decode_step(*(_np(t) for t in tk), Sr)
        assert_close(o, o_ref, TOL[dtype], f"step {i} o")
    gdr2_sync_status()
    assert_close(Sg, Sr, TOL[dtype], "state after 12 steps")


def test_prefill_then_decode_matches_longer_prefill():
    """Decoding token T after a prefill of T tokens equals a prefill of T + 1 tokens."""
    x = I.make_forward_inputs(B=2, H=16, T=97, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=8)
    d = x.to("cuda")
    o_all, S_all, _ = gdr2_forward(d.q, d.k, d.v, d.log_alpha, d.b, d.w, None)
    _, S_pre, _ = gdr2_forward(*(t[:, :96].contiguous() for t in (d.q, d.k, d.v, d.log_alpha, d.b, d.w)), None)
    o_dec = gdr2_decode_step(*(t[:, 96].contiguous() for t in (d.q, d.k, d.v, d.log_alpha, d.b, d.w)), S_pre)
    gdr2_sync_status()
    assert_close(o_dec, _np(o_all[:, 96]), 2e-2, "decoded token")
    assert_close(S_pre, _np(S_all), 2e-2, "state after decoding")


def test_decode_reset_token():
    """alpha = 0 (log alpha = -inf) wipes the state: S = k z^T."""
    S, toks = I.make_decode_inputs(N=4, H=2, dk=128, dv=128, dtype=torch.float32, seed=9, steps=1)
    q, k, v, la, b, w = toks[0]
    la = torch.full_like(la, float("-inf"))
    Sg = S.cuda()
    o = gdr2_decode_step(q.cuda(), k.cuda(), v.cuda(), la.cuda(), b.cuda(), w.cuda(), Sg)
    o_ref, S_ref = oracle.decode_step(_np(q), _np(k), _np(v), _np(la), _np(b), _np(w), S.double().numpy())
    gdr2_sync_status()
    assert_close(Sg, S_ref, 1e-5, "reset state")
    assert_close(o, o_ref, 1e-5, "reset output")


@pytest.mark.slow
def test_full_size_512_steps_sampled_heads():
    """256 sequences x 16 heads, d = 128, fp32 state (256 MiB), 512 consecutive steps.

    Every step's tokens are drawn on the device from a seeded generator; the
    oracle replays the sampled (sequence, head) pairs on their copies.
    """
    cfg = I.DECODE_1P3B
    N, H, dk, dv, steps = cfg["N"], cfg["H"], cfg["dk"], cfg["dv"], cfg["steps"]
    gen = torch.Generator(device="cuda").manual_seed(cfg["seed"])
    S = torch.randn((N, H, dk, dv), device="cuda", generator=gen) * cfg["state_std"]
    pn = torch.tensor([0, 17, 128, 255], device="cuda")
    ph = torch.tensor([0, 5, 9, 15], device="cuda")
    Sr = _np(S[pn, ph])[None]  # [1, P, dk, dv]
    for step in range(steps):
        tk = I.make_token_inputs((N, H, dk), (N, H, dv), cfg["dtype"], cfg["decay_shift"], gen)
        o = gdr2_decode_step(*tk, S)
        sel = [_np(t[pn, ph])[None] for t in tk]
        o_ref, Sr = oracle.decode_step(*sel, Sr)
        assert_close(_np(o[pn, ph])[None], o_ref, TOL[cfg["dtype"]], f"step {step} o")
    gdr2_sync_status()
    S_sel = _np(S[pn, ph])[None]
    assert_close(S_sel, Sr, TOL[cfg["dtype"]], "state after 512 steps")
    assert torch.isfinite(S).all()
