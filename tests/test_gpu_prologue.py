"""GPU parity of the block prologue (short causal convolution + SiLU + per-head L2 norm,
and the decay and gate activations) against the fp64 oracle (Gated DeltaNet-2 note,
sec. 3, block data-flow paragraph), and of the whole block data flow: prologue, mixer
and output epilogue against the oracle's chain."""
import numpy as np
import pytest
import torch

import oracle
from oracle import block as OB
from gated_delta_rule_wy_b200 import (gdr2_block_prologue, gdr2_forward, gdr2_gate_activations,
                                      gdr2_short_conv_silu, gdr2_sync_status)
from gated_delta_rule_wy_b200 import inputs as I
from parity import TOL, assert_close, assert_epilogue_close

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().to("cpu", torch.float64).numpy()


def _expected_state(x, W, state):
    """The state after the call is a copy of inputs: exact in the input dtype."""
    return torch.from_numpy(OB.conv_state_after(_np(x), W, None if state is None else _np(state)))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("W", [4, 2, 1])
@pytest.mark.parametrize("l2", [True, False])
def test_dense_conv_matches_the_oracle(dtype, d, W, l2):
    N, T, H = 2, 77, 3  # 77 tokens: two 32-token runs and a ragged one
    x, wgt, st = I.make_conv_inputs((N, T, H, d), W, dtype, seed=111)
    y, s_out = gdr2_short_conv_silu(x.cuda(), wgt.cuda(), st.cuda(), l2norm=l2, eps=1e-6, final_state=True)
    gdr2_sync_status()
    xr = _np(x).reshape(N, T, H * d)
    sr = _np(st).reshape(N, W - 1, H * d)
    y_ref, s_ref = OB.short_conv_silu(xr, _np(wgt), sr, l2norm=l2, eps=1e-6, heads=H)
    assert_close(y.reshape(N, T, H * d), y_ref, TOL[dtype], f"y (W={W}, d={d}, l2={l2})")
    assert torch.equal(s_out.cpu(), torch.from_numpy(s_ref.reshape(N, W - 1, H, d)).to(dtype))


def test_without_a_state_the_past_is_zero():
    x, wgt, _ = I.make_conv_inputs((1, 40, 2, 128), 4, torch.bfloat16, seed=112)
    y, _ = gdr2_short_conv_silu(x.cuda(), wgt.cuda(), None)
    gdr2_sync_status()
    y_ref, _ = OB.short_conv_silu(_np(x).reshape(1, 40, 256), _np(wgt))
    assert_close(y.reshape(1, 40, 256), y_ref, TOL[torch.bfloat16], "y without a state")


@pytest.mark.parametrize("l2", [True, False])
def test_packed_sequences_convolve_on_their_own(l2):
    lens = [0, 5, 1, 70, 2, 0, 40]  # empty, short (< W - 1), across 32-token runs
    T, H, d, W = sum(lens), 2, 128, 4
    cu = np.concatenate([[0], np.cumsum(lens)])
    x, wgt, _ = I.make_conv_inputs((T, H, d), W, torch.bfloat16, seed=113)
    _, _, sts = I.make_conv_inputs((len(lens), 1, H, d), W, torch.bfloat16, seed=114)
    y, s_out = gdr2_short_conv_silu(x.cuda(), wgt.cuda(), sts.cuda(), l2norm=l2,
                                    cu_seqlens=torch.tensor(cu, dtype=torch.int32, device="cuda"), final_state=True)
    gdr2_sync_status()
    y_ref, s_ref = OB.short_conv_silu(_np(x).reshape(1, T, H * d), _np(wgt), l2norm=l2, heads=H, cu_seqlens=cu,
                                      states=_np(sts).reshape(len(lens), W - 1, H * d))
    assert_close(y.reshape(1, T, H * d), y_ref, TOL[torch.bfloat16], "packed y")
    assert torch.equal(s_out.cpu(), torch.from_numpy(s_ref.reshape(len(lens), W - 1, H, d)).to(torch.bfloat16))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_steps_in_place_equal_one_call(dtype):
    """Ten one-token calls, the state updated in place, give the bits of one ten-token call."""
    N, T, H, d, W = 4, 10, 2, 128, 4
    x, wgt, st = I.make_conv_inputs((N, T, H, d), W, dtype, seed=115)
    xc, wc = x.cuda(), wgt.cuda()
    y_all, s_all = gdr2_short_conv_silu(xc, wc, st.cuda(), l2norm=True, final_state=True)
    s = st.cuda().clone()
    ys = []
    for t in range(T):
        yt, _ = gdr2_short_conv_silu(xc[:, t:t + 1].contiguous(), wc, s, l2norm=True, state_out=s)
        ys.append(yt)
    gdr2_sync_status()
    assert torch.equal(torch.cat(ys, 1), y_all) and torch.equal(s, s_all)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("shape", [(2, 100, 3, 128), (2, 101, 3)])  # vector gates; scalar gates (ragged count)
def test_gate_activations_match_the_oracle(dtype, shape):
    g = torch.Generator().manual_seed(116)
    a = (torch.randn(shape, generator=g) * 4 + 2).to(dtype)
    b = (torch.randn(shape, generator=g) * 4).to(dtype)
    w = (torch.randn(shape, generator=g) * 4).to(dtype)
    la, bo, wo = gdr2_gate_activations(a.cuda(), b.cuda(), w.cuda())
    gdr2_sync_status()
    assert la.dtype == torch.float32 and bo.dtype == dtype
    assert_close(la, OB.neg_softplus(_np(a)), 1e-5, "log alpha")
    assert_close(bo, OB.sigmoid(_np(b)), TOL[dtype] / 4, "b")
    assert_close(wo, OB.sigmoid(_np(w)), TOL[dtype] / 4, "w")
    la2, _, _ = gdr2_gate_activations(a.cuda())  # one branch alone
    gdr2_sync_status()
    assert torch.equal(la2, la)


def test_block_data_flow_end_to_end():
    """Prologue -> mixer -> output epilogue on the GPU against the oracle's same chain from
    the same projections (B=1, H=2, T=200, d=128, bf16)."""
    B, T, H, d, W = 1, 200, 2, 128, 4
    p = I.make_prologue_inputs(B, T, H, d, d, W, torch.bfloat16, seed=117)
    g, wt = I.make_epilogue_inputs((B, T, H, d), d, seed=118)
    dv = {k: v.cuda() for k, v in p.items()}
    q, k, v, la, b, w, _ = gdr2_block_prologue(dv["xq"], dv["xk"], dv["xv"], dv["conv_q"], dv["conv_k"],
                                               dv["conv_v"], dv["a"], dv["b"], dv["w"])
    y, S_T, _ = gdr2_forward(q, k, v, la, b, w, None, out_gate=g.cuda(), norm_weight=wt.cuda())
    gdr2_sync_status()
    n = {kk: _np(vv) for kk, vv in p.items()}
    rs = lambda a_: a_.reshape(B, T, H * d)  # noqa: E731
    back = lambda a_: a_.reshape(B, T, H, d)  # noqa: E731
    qr, _ = OB.short_conv_silu(rs(n["xq"]), n["conv_q"], l2norm=True, heads=H)
    kr, _ = OB.short_conv_silu(rs(n["xk"]), n["conv_k"], l2norm=True, heads=H)
    vr, _ = OB.short_conv_silu(rs(n["xv"]), n["conv_v"], heads=H)
    o_ref, S_ref = oracle.forward(back(qr), back(kr), back(vr), OB.neg_softplus(n["a"]), OB.sigmoid(n["b"]),
                                  OB.sigmoid(n["w"]))
    gn, wn = _np(g), _np(wt)
    y_ref = OB.output_norm_gate(o_ref, gn, wn, 1e-6)
    assert_epilogue_close(y, y_ref, o_ref, gn, wn, 1e-6, TOL[torch.bfloat16], "block y")
    assert_close(S_T, S_ref, TOL[torch.bfloat16], "block S_T")


@pytest.mark.slow
def test_full_size_1p3b_layer_prologue_sampled_heads():
    """B=4 H=16 T=4096 d=128 bf16 width 4, the benchmarked launch; oracle on sampled (b, h)."""
    B, T, H, d, W = 4, 4096, 16, 128, 4
    p = I.make_prologue_inputs(B, T, H, d, d, W, torch.bfloat16, seed=1010)
    dv = {k: v.cuda() for k, v in p.items()}
    q, k, v, la, b, w, _ = gdr2_block_prologue(dv["xq"], dv["xk"], dv["xv"], dv["conv_q"], dv["conv_k"],
                                               dv["conv_v"], dv["a"], dv["b"], dv["w"])
    gdr2_sync_status()
    for (bb, h) in [(0, 0), (1, 9), (3, 15)]:
        for name, y, l2 in (("q", q, True), ("k", k, True), ("v", v, False)):
            xs = _np(p["x" + name][bb:bb + 1, :, h])                       # [1, T, d]
            ws = _np(p["conv_" + name].reshape(H, d, W)[h])               # [d, W]
            y_ref, _ = OB.short_conv_silu(xs, ws, l2norm=l2, heads=1)
            assert_close(y[bb:bb + 1, :, h], y_ref, TOL[torch.bfloat16], f"{name}[b={bb},h={h}]")
        assert_close(la[bb, :, h], OB.neg_softplus(_np(p["a"][bb, :, h])), 1e-5, f"log alpha[b={bb},h={h}]")
        assert_close(b[bb, :, h], OB.sigmoid(_np(p["b"][bb, :, h])), TOL[torch.bfloat16] / 4, f"b[b={bb},h={h}]")
        assert_close(w[bb, :, h], OB.sigmoid(_np(p["w"][bb, :, h])), TOL[torch.bfloat16] / 4, f"w[b={bb},h={h}]")


def test_width_three_and_fp32_packed():
    x, wgt, st = I.make_conv_inputs((2, 45, 2, 64), 3, torch.bfloat16, seed=120)
    y, s_out = gdr2_short_conv_silu(x.cuda(), wgt.cuda(), st.cuda(), l2norm=True, final_state=True)
    gdr2_sync_status()
    y_ref, s_ref = OB.short_conv_silu(_np(x).reshape(2, 45, 128), _np(wgt), _np(st).reshape(2, 2, 128), l2norm=True,
                                      heads=2)
    assert_close(y.reshape(2, 45, 128), y_ref, TOL[torch.bfloat16], "W=3 y")
    assert torch.equal(s_out.cpu(), torch.from_numpy(s_ref.reshape(2, 2, 2, 64)).to(torch.bfloat16))
    lens = [33, 0, 2, 40]
    cu = np.concatenate([[0], np.cumsum(lens)])
    xp, wp, _ = I.make_conv_inputs((sum(lens), 2, 128), 4, torch.float32, seed=121)
    _, _, sp = I.make_conv_inputs((len(lens), 1, 2, 128), 4, torch.float32, seed=122)
    y, s_out = gdr2_short_conv_silu(xp.cuda(), wp.cuda(), sp.cuda(), cu_seqlens=torch.tensor(cu, dtype=torch.int32,
                                    device="cuda"), final_state=True)
    gdr2_sync_status()
    y_ref, s_ref = OB.short_conv_silu(_np(xp).reshape(1, -1, 256), _np(wp), cu_seqlens=cu,
                                      states=_np(sp).reshape(len(lens), 3, 256))
    assert_close(y.reshape(1, -1, 256), y_ref, TOL[torch.float32], "fp32 packed y")
    assert torch.equal(s_out.cpu(), torch.from_numpy(s_ref.reshape(len(lens), 3, 2, 128)).float())


def test_no_tokens_pass_the_state_through():
    _, wgt, st = I.make_conv_inputs((2, 1, 2, 128), 4, torch.bfloat16, seed=123)
    x = torch.empty((2, 0, 2, 128), dtype=torch.bfloat16, device="cuda")
    y, s_out = gdr2_short_conv_silu(x, wgt.cuda(), st.cuda(), final_state=True)  # dense, T = 0
    gdr2_sync_status()
    assert y.numel() == 0 and torch.equal(s_out.cpu(), st)
    xp = torch.empty((0, 2, 128), dtype=torch.bfloat16, device="cuda")
    cu = torch.zeros(3, dtype=torch.int32, device="cuda")  # two empty packed sequences
    _, s_out = gdr2_short_conv_silu(xp, wgt.cuda(), st.cuda(), cu_seqlens=cu, final_state=True)
    gdr2_sync_status()
    assert torch.equal(s_out.cpu(), st)
    _, s_zero = gdr2_short_conv_silu(xp, wgt.cuda(), None, cu_seqlens=cu, final_state=True)
    gdr2_sync_status()
    assert torch.count_nonzero(s_zero) == 0
