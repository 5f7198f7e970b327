"""The backward entry point that allocates no device memory (needs a B200).

Some callers cannot call cudaMalloc: for example a serving engine that has
reserved nearly all device memory for its own pool (a fresh allocation would
fail or fragment it, and cudaFree synchronises the device), or a host module
that only receives device pointers from another runtime. For them the library
exports gdr2_backward_noalloc, which keeps its scratch in a fixed device array
inside the library instead of a caller workspace. This test calls it through
the C ABI twice in a row, on different problems, and checks each result
against gdr2_backward (the workspace entry point) within the parity
tolerances the other tests use. It lives in its own file, collected last.
"""
import pytest
import torch

from gated_delta_rule_wy_b200 import gdr2_backward, gdr2_backward_noalloc, gdr2_forward, gdr2_sync_status
from gated_delta_rule_wy_b200 import inputs as I

pytestmark = pytest.mark.gpu

GRADS = ("dq", "dk", "dv", "dlog_alpha", "db", "dw", "dS0")
TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def _rel(a, b):
    a, b = a.double(), b.double()
    return float((a - b).abs().max() / b.abs().max().clamp_min(1e-30))


@pytest.mark.parametrize("order", ["bf16_then_f32", "f32_then_bf16"])
def test_noalloc_backward_matches_workspace_backward_twice(order):
    cases = [dict(B=1, T=150, H=3, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=61,
                  with_S0=True, use_saved=False),
             dict(B=2, T=97, H=2, dk=64, dv=128, dtype=torch.float32, decay_shift=0.0, seed=62,
                  with_S0=True, use_saved=True)]
    if order == "f32_then_bf16":
        cases = cases[::-1]
    for call, cfg in enumerate(cases):
        use_saved = cfg.pop("use_saved")
        x = I.make_forward_inputs(**cfg).to("cuda")
        B, T, H, dk, dv = cfg["B"], cfg["T"], cfg["H"], cfg["dk"], cfg["dv"]
        dO = I.make_upstream_grad(B, T, H, dv, cfg["seed"], dtype=cfg["dtype"]).cuda()
        dST = torch.randn((B, H, dk, dv), generator=torch.Generator().manual_seed(cfg["seed"])).cuda()
        saved = None
        if use_saved:
            _, _, saved = gdr2_forward(x.q, x.k, x.v, x.log_alpha, x.b, x.w, x.S0, save_states=True)
        ref = gdr2_backward(x.q, x.k, x.v, x.log_alpha, x.b, x.w, dO, x.S0, dST, saved)
        got = gdr2_backward_noalloc(x.q, x.k, x.v, x.log_alpha, x.b, x.w, dO, x.S0, dST, saved)
        gdr2_sync_status()
        for n in GRADS:
            e = _rel(got[n], ref[n])
            assert e <= TOL[cfg["dtype"]], f"call {call + 1} ({cfg['dtype']}): {n} differs by {e:.2e}"
