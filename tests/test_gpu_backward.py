"""GPU parity of gdr2_backward against the oracle's reverse mode (needs a B200)."""
import pytest
import torch

import oracle
from gated_delta_rule_wy_b200 import gdr2_backward, gdr2_forward, gdr2_sync_status
from gated_delta_rule_wy_b200 import inputs as I
from parity import TOL, assert_close, head_slice

pytestmark = pytest.mark.gpu

GRADS = ("dq", "dk", "dv", "dlog_alpha", "db", "dw", "dS0")


def _case(B, T, H, dk, dv, dtype, seed, with_S0=True, with_dST=True):
    x = I.make_forward_inputs(B=B, H=H, T=T, dk=dk, dv=dv, dtype=dtype, decay_shift=2.0, seed=seed,
                              with_S0=with_S0)
    dO = I.make_upstream_grad(B, T, H, dv, seed, dtype=dtype)
    dST = torch.randn((B, H, dk, dv), generator=torch.Generator().manual_seed(seed + 1)) if with_dST else None
    return x, dO, dST


def _oracle(x, dO, dST):
    n = x.as_numpy64()
    return oracle.backward(n["q"], n["k"], n["v"], n["log_alpha"], n["b"], n["w"],
                           dO.double().numpy(), S0=n["S0"],
                           dS_T=None if dST is None else dST.double().numpy())


def _gpu(x, dO, dST, use_saved):
    d = x.to("cuda")
    saved = None
    if use_saved:
        _, _, saved = gdr2_forward(d.q, d.k, d.v, d.log_alpha, d.b, d.w, d.S0, save_states=True)
    g = gdr2_backward(d.q, d.k, d.v, d.log_alpha, d.b, d.w, dO.cuda(), d.S0,
                      None if dST is None else dST.cuda(), saved)
    gdr2_sync_status()
    return g


@pytest.mark.parametrize("use_saved", [False, True])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 64), (64, 128), (128, 128)])
def test_f32_ragged(dk, dv, use_saved):
    x, dO, dST = _case(1, 100, 2, dk, dv, torch.float32, seed=30 + dk + dv)
    g = _gpu(x, dO, dST, use_saved)
    ref = _oracle(x, dO, dST)
    for n in GRADS:
        assert_close(g[n], ref[n], 1e-4, f"fp32 {n}")


@pytest.mark.parametrize("use_saved", [False, True])
def test_bf16_t256_slice_of_backward_workload(use_saved):
    """B=2 H=16 T=256 d=128 bf16 (a T=256 slice of the backward workload), bound 2e-2."""
    x, dO, _ = _case(2, 256, 16, 128, 128, torch.bfloat16, seed=I.BWD_1P3B_BF16["seed"], with_S0=False,
                     with_dST=False)
    g = _gpu(x, dO, None, use_saved)
    ref = _oracle(x, dO, None)
    for n in GRADS:
        assert_close(g[n], ref[n], TOL[torch.bfloat16], f"bf16 {n}")


def test_short_sequences():
    for T in (1, 3, 64, 65):
        x, dO, dST = _case(1, T, 1, 128, 128, torch.float32, seed=40 + T)
        g = _gpu(x, dO, dST, False)
        ref = _oracle(x, dO, dST)
        for n in GRADS:
            assert_close(g[n], ref[n], 1e-4, f"T={T} {n}")


@pytest.mark.slow
def test_full_size_backward_sampled_heads():
    """B=2 H=16 T=4096 d=128 bf16 with saved chunk states; oracle on two heads."""
    cfg = I.BWD_1P3B_BF16
    x, dO, _ = _case(cfg["B"], cfg["T"], cfg["H"], 128, 128, torch.bfloat16, seed=cfg["seed"], with_S0=False,
                     with_dST=False)
    g = _gpu(x, dO, None, True)
    n = x.as_numpy64()
    dOn = dO.double().numpy()
    for (b, h) in [(0, 3), (1, 12)]:
        args = [head_slice(n[f], b, h) for f in ("q", "k", "v", "log_alpha", "b", "w")]
        ref = oracle.backward(*args, head_slice(dOn, b, h))
        for name in GRADS[:-1]:
            assert_close(g[name][b:b + 1, :, h:h + 1], ref[name], TOL[torch.bfloat16], f"{name}[b={b},h={h}]")
        assert_close(g["dS0"][b:b + 1, h:h + 1], ref["dS0"], TOL[torch.bfloat16], f"dS0[b={b},h={h}]")
