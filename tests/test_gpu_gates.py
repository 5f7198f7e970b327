"""Scalar gates (one value per token-head) on the GPU.

A scalar erase or write gate is the vector gate with that value in every channel, so every
path must give exactly what it gives for the broadcast vector (same arithmetic, same bits),
and the KDA / Gated DeltaNet setting b = w = beta must match the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_wy_b200 import gdr2_decode_step, gdr2_forward, gdr2_forward_varlen, gdr2_sync_status
from gated_delta_rule_wy_b200 import inputs as I
from parity import TOL, assert_close

pytestmark = pytest.mark.gpu

MODES = {"scalar_b": (True, False), "scalar_w": (False, True), "both": (True, True)}


def _scalar_gates(shape, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.sigmoid(torch.randn(shape, generator=g)).to(dtype),
            torch.sigmoid(torch.randn(shape, generator=g)).to(dtype))


def _vec(s, d):
    return s[..., None].expand(*s.shape, d).contiguous()


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("dtype, d, T, la_shift", [(torch.bfloat16, 128, 200, 0.0),   # tensor-core path
                                                  (torch.bfloat16, 128, 130, -30.0),  # its exact path
                                                  (torch.float32, 64, 150, 0.0)])     # SIMT path
def test_forward_scalar_gates_equal_broadcast_vectors(mode, dtype, d, T, la_shift):
    sb_on, sw_on = MODES[mode]
    x = I.make_forward_inputs(B=2, H=3, T=T, dk=d, dv=d, dtype=dtype, decay_shift=2.0, seed=81, with_S0=True)
    sb, sw = _scalar_gates((2, T, 3), dtype, 82)
    b = sb if sb_on else x.b
    w = sw if sw_on else x.w
    la = x.log_alpha + la_shift
    d_ = x.to("cuda")
    args_s = [d_.q, d_.k, d_.v, la.cuda(), b.cuda(), w.cuda(), d_.S0]
    args_v = [d_.q, d_.k, d_.v, la.cuda(), (_vec(sb, d) if sb_on else x.b).cuda(),
              (_vec(sw, d) if sw_on else x.w).cuda(), d_.S0]
    o_s, S_s, _ = gdr2_forward(*args_s)
    o_v, S_v, _ = gdr2_forward(*args_v)
    gdr2_sync_status()
    assert torch.equal(o_s, o_v), f"{mode}: o differs from the broadcast-vector run"
    assert torch.equal(S_s, S_v), f"{mode}: S_T differs from the broadcast-vector run"


@pytest.mark.parametrize("mode", list(MODES))
def test_packed_sequences_with_scalar_gates(mode):
    sb_on, sw_on = MODES[mode]
    lens = [0, 70, 1, 128, 33]
    T = sum(lens)
    x = I.make_forward_inputs(B=1, H=2, T=T, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=83)
    sb, sw = _scalar_gates((1, T, 2), torch.bfloat16, 84)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    d_ = x.to("cuda")
    bs = (sb if sb_on else x.b).cuda()
    ws = (sw if sw_on else x.w).cuda()
    bv = (_vec(sb, 128) if sb_on else x.b).cuda()
    wv = (_vec(sw, 128) if sw_on else x.w).cuda()
    o_s, S_s, _ = gdr2_forward_varlen(d_.q, d_.k, d_.v, d_.log_alpha, bs, ws, cu)
    o_v, S_v, _ = gdr2_forward_varlen(d_.q, d_.k, d_.v, d_.log_alpha, bv, wv, cu)
    gdr2_sync_status()
    assert torch.equal(o_s, o_v) and torch.equal(S_s, S_v)


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_scalar_gates_equal_broadcast_vectors(mode, dtype):
    sb_on, sw_on = MODES[mode]
    N, H, d = 8, 4, 128
    g = torch.Generator(device="cuda").manual_seed(85)
    q, k, v, la, b, w = I.make_token_inputs((N, H, d), (N, H, d), dtype, 2.0, g)
    sb, sw = (t.cuda() for t in _scalar_gates((N, H), dtype, 86))
    S = torch.randn((N, H, d, d), device="cuda", generator=g) * 0.05
    S2 = S.clone()
    o_s = gdr2_decode_step(q, k, v, la, sb if sb_on else b, sw if sw_on else w, S)
    o_v = gdr2_decode_step(q, k, v, la, _vec(sb, d) if sb_on else b, _vec(sw, d) if sw_on else w, S2)
    gdr2_sync_status()
    assert torch.equal(o_s, o_v) and torch.equal(S, S2)


def test_kda_gates_match_the_oracle():
    """b = w = beta per token-head (the Gated DeltaNet / KDA gates) on the tensor-core path."""
    B, H, T = 1, 2, 256
    x = I.make_forward_inputs(B=B, H=H, T=T, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=87,
                              with_S0=True)
    beta, _ = _scalar_gates((B, T, H), torch.bfloat16, 88)
    d_ = x.to("cuda")
    o, S_T, _ = gdr2_forward(d_.q, d_.k, d_.v, d_.log_alpha, beta.cuda(), beta.cuda(), d_.S0)
    gdr2_sync_status()
    n = x.as_numpy64()
    bv = np.repeat(beta.double().numpy()[..., None], 128, axis=-1)
    o_ref, S_ref = oracle.forward(n["q"], n["k"], n["v"], n["log_alpha"], bv, bv, S0=n["S0"])
    assert_close(o, o_ref, TOL[torch.bfloat16], "KDA gates: o")
    assert_close(S_T, S_ref, TOL[torch.bfloat16], "KDA gates: S_T")


def _oracle_backward(x, b_vec, w_vec, dO, dST):
    n = x.as_numpy64()
    return oracle.backward(n["q"], n["k"], n["v"], n["log_alpha"], b_vec, w_vec, dO.double().numpy(), S0=n["S0"],
                           dS_T=None if dST is None else dST.double().numpy())


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("shape", [(2, 16, 256, False), (1, 3, 150, True)])
def test_backward_scalar_gates_match_the_oracle(mode, shape):
    """Scalar erase and/or write gates through the tensor-core backward (the first shape is
    the T = 256 slice of the backward workload, the second a ragged one with S0 and dS_T):
    each gradient against the oracle's for the broadcast vector gates, a scalar gate's
    gradient against the sum of the vector gradient over its channels; the other
    gradients equal those of the broadcast-vector call."""
    from gated_delta_rule_wy_b200 import gdr2_backward

    B, H, T, with_state = shape
    sb_on, sw_on = MODES[mode]
    x = I.make_forward_inputs(B=B, H=H, T=T, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=89,
                              with_S0=with_state)
    sb, sw = _scalar_gates((B, T, H), torch.bfloat16, 90)
    dO = I.make_upstream_grad(B, T, H, 128, 91, dtype=torch.bfloat16)
    dST = torch.randn((B, H, 128, 128), generator=torch.Generator().manual_seed(92)) if with_state else None
    bv = _vec(sb, 128) if sb_on else x.b
    wv = _vec(sw, 128) if sw_on else x.w
    d_ = x.to("cuda")
    dev = lambda t: None if t is None else t.cuda()  # noqa: E731
    g = gdr2_backward(d_.q, d_.k, d_.v, d_.log_alpha, dev(sb if sb_on else x.b), dev(sw if sw_on else x.w),
                      dO.cuda(), d_.S0, dev(dST))
    gv = gdr2_backward(d_.q, d_.k, d_.v, d_.log_alpha, bv.cuda(), wv.cuda(), dO.cuda(), d_.S0, dev(dST))
    gdr2_sync_status()
    assert g["db"].shape == ((B, T, H) if sb_on else (B, T, H, 128))
    assert g["dw"].shape == ((B, T, H) if sw_on else (B, T, H, 128))
    ref = _oracle_backward(x, bv.double().numpy(), wv.double().numpy(), dO, dST)
    for name in ("dq", "dk", "dv", "dlog_alpha", "db", "dw", "dS0"):
        r = ref[name]
        if (name == "db" and sb_on) or (name == "dw" and sw_on):
            r = r.sum(axis=-1)
        assert_close(g[name], r, TOL[torch.bfloat16], f"{mode} {shape}: {name}")
    for name in ("dq", "dk", "dv", "dlog_alpha", "dS0"):
        assert torch.equal(g[name], gv[name]), f"{mode} {shape}: {name} differs from the broadcast-vector call"


def test_backward_scalar_gates_need_the_tensor_core_path():
    from gated_delta_rule_wy_b200 import binding, gdr2_backward

    x = I.make_forward_inputs(B=1, H=2, T=70, dk=64, dv=64, dtype=torch.float32, seed=93).to("cuda")
    sb, _ = _scalar_gates((1, 70, 2), torch.float32, 94)
    dO = I.make_upstream_grad(1, 70, 2, 64, 95).cuda()
    with pytest.raises(binding.GDR2Error, match="UNSUPPORTED"):
        gdr2_backward(x.q, x.k, x.v, x.log_alpha, sb.cuda(), x.w, dO)
