"""The backward entry point that allocates no device memory (needs a B200).

Some callers cannot call cudaMalloc: for example a serving engine that has
reserved nearly all device memory for its own pool (a fresh allocation would
fail or fragment it, and cudaFree synchronises the device), or a host module
that only receives device pointers from another runtime. For them the library
exports gdr2_backward_noalloc, which keeps its scratch in a fixed device array
inside the library instead of a caller workspace. This test calls it through
the C ABI several times in a row, on different problems, and checks each result
against gdr2_backward (the workspace entry point) and against the fp64 oracle,
within the parity tolerances the other tests use. Each later call finds the
array holding the previous call's contents; one of them recomputes the chunk
states itself (no saved states), the part of the array a larger call filled
just before. It lives in its own file, collected last.
"""
import pytest
import torch

import oracle
from gated_delta_rule_wy_b200 import gdr2_backward, gdr2_backward_noalloc, gdr2_forward, gdr2_sync_status
from gated_delta_rule_wy_b200 import inputs as I

pytestmark = pytest.mark.gpu

GRADS = ("dq", "dk", "dv", "dlog_alpha", "db", "dw", "dS0")
TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def _rel(a, b):
    a, b = a.double().cpu(), torch.as_tensor(b).double().cpu()
    return float((a - b).abs().max() / b.abs().max().clamp_min(1e-30))


def _run(cfg):
    cfg = dict(cfg)
    use_saved = cfg.pop("use_saved")
    xc = I.make_forward_inputs(**cfg)
    x = xc.to("cuda")
    B, T, H, dk, dv = cfg["B"], cfg["T"], cfg["H"], cfg["dk"], cfg["dv"]
    dOc = I.make_upstream_grad(B, T, H, dv, cfg["seed"], dtype=cfg["dtype"])
    dSTc = torch.randn((B, H, dk, dv), generator=torch.Generator().manual_seed(cfg["seed"]))
    dO, dST = dOc.cuda(), dSTc.cuda()
    saved = None
    if use_saved:
        _, _, saved = gdr2_forward(x.q, x.k, x.v, x.log_alpha, x.b, x.w, x.S0, save_states=True)
    ref = gdr2_backward(x.q, x.k, x.v, x.log_alpha, x.b, x.w, dO, x.S0, dST, saved)
    got = gdr2_backward_noalloc(x.q, x.k, x.v, x.log_alpha, x.b, x.w, dO, x.S0, dST, saved)
    gdr2_sync_status()
    n = xc.as_numpy64()
    exact = oracle.backward(n["q"], n["k"], n["v"], n["log_alpha"], n["b"], n["w"], dOc.double().numpy(),
                            S0=n["S0"], dS_T=dSTc.double().numpy())
    tol = TOL[cfg["dtype"]]
    for g in GRADS:
        e = _rel(got[g], ref[g])
        assert e <= tol, f"{cfg['dtype']} T={T}: {g} differs from gdr2_backward by {e:.2e}"
        e = _rel(got[g], exact[g])
        assert e <= tol, f"{cfg['dtype']} T={T}: {g} differs from the oracle by {e:.2e}"


LARGE = dict(B=2, T=300, H=4, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=63, with_S0=True,
             use_saved=False)
CASES = [dict(B=1, T=150, H=3, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=61,
              with_S0=True, use_saved=False),
         dict(B=2, T=97, H=2, dk=64, dv=128, dtype=torch.float32, decay_shift=0.0, seed=62,
              with_S0=True, use_saved=True)]


@pytest.mark.parametrize("order", ["bf16_then_f32", "f32_then_bf16"])
def test_noalloc_backward_matches_workspace_backward_and_oracle(order):
    cases = CASES if order == "bf16_then_f32" else CASES[::-1]
    for cfg in cases:
        _run(cfg)


def test_noalloc_backward_recomputes_states_over_a_larger_calls_scratch():
    """A larger call fills the chunk-state region; then T = 200 without saved states (the
    kernel recomputes the states entering each chunk into that region) reads only what it
    wrote itself."""
    _run(LARGE)
    _run(dict(B=1, T=200, H=2, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=64, with_S0=True,
              use_saved=False))
