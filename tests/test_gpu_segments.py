"""GPU parity of the segmented forward (sequences cut into segments run side by side; the
entering states from gdr2_segment_states) against the fp64 oracle over whole sequences."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_wy_b200 import (gdr2_forward, gdr2_forward_segmented, gdr2_segment_states,
                                      gdr2_sync_status)
from gated_delta_rule_wy_b200 import inputs as I
from parity import TOL, assert_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dk, dv", [(128, 128), (128, 64), (64, 64)])
def test_segment_states_scan(dk, dv):
    B, G, H = 2, 5, 3
    g = torch.Generator().manual_seed(141)
    A = torch.randn((B, G, H, dk, dk), generator=g) / dk ** 0.5
    Bst = torch.randn((B, G, H, dk, dv), generator=g)
    S0 = torch.randn((B, H, dk, dv), generator=g)
    starts, S_T = gdr2_segment_states(A.cuda(), Bst.cuda(), S0.cuda())
    gdr2_sync_status()
    S = S0.double()
    for gg in range(G):
        assert_close(starts[:, gg], S.numpy(), 1e-5, f"entering state {gg}")
        S = A[:, gg].double() @ S + Bst[:, gg].double()
    assert_close(S_T, S.numpy(), 1e-5, "final state")


@pytest.mark.parametrize("dtype, d, T, G", [(torch.bfloat16, 128, 512, 4),   # tensor-core forward
                                            (torch.bfloat16, 128, 384, 3),   # segments of 128 tokens
                                            (torch.float32, 64, 256, 4)])    # CUDA-core forward
def test_segmented_forward_matches_the_oracle(dtype, d, T, G):
    x = I.make_forward_inputs(B=2, H=2, T=T, dk=d, dv=d, dtype=dtype, decay_shift=2.0 if dtype == torch.bfloat16
                              else 0.0, seed=142, with_S0=True)
    dx = x.to("cuda")
    o, S_T = gdr2_forward_segmented(dx.q, dx.k, dx.v, dx.log_alpha, dx.b, dx.w, dx.S0, segments=G)
    gdr2_sync_status()
    n = x.as_numpy64()
    o_ref, S_ref = oracle.forward(n["q"], n["k"], n["v"], n["log_alpha"], n["b"], n["w"], S0=n["S0"])
    assert_close(o, o_ref, TOL[dtype], f"o (G={G})")
    assert_close(S_T, S_ref, TOL[dtype], f"S_T (G={G})")


def test_segmented_equals_plain_forward_with_scalar_gates():
    """b = w = beta per token-head (the KDA / Gated DeltaNet gates), against the plain forward."""
    B, H, T, G = 1, 2, 256, 4
    x = I.make_forward_inputs(B=B, H=H, T=T, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=143)
    beta = torch.sigmoid(torch.randn((B, T, H), generator=torch.Generator().manual_seed(144))).to(torch.bfloat16)
    d = x.to("cuda")
    o_s, S_s = gdr2_forward_segmented(d.q, d.k, d.v, d.log_alpha, beta.cuda(), beta.cuda(), segments=G)
    o_p, S_p, _ = gdr2_forward(d.q, d.k, d.v, d.log_alpha, beta.cuda(), beta.cuda())
    gdr2_sync_status()
    assert_close(o_s, o_p.double().cpu().numpy(), TOL[torch.bfloat16], "o vs the plain forward")
    assert_close(S_s, S_p.double().cpu().numpy(), TOL[torch.bfloat16], "S_T vs the plain forward")
    assert np.isfinite(o_s.float().cpu().numpy()).all()
