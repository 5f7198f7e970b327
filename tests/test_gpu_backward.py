"""GPU parity of gdr2_backward against the oracle's reverse mode (needs a B200).

bf16 inputs at dk = dv = 128 run the chunkwise tensor-core backward; fp32 inputs and the
other head sizes run the token-level kernel."""
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


@pytest.mark.parametrize("use_saved", [False, True])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
def test_bf16_ragged_with_state_and_state_gradient(T, use_saved):
    """Tensor-core path: a partial last chunk, an initial state and an upstream dS_T."""
    x, dO, dST = _case(2, T, 3, 128, 128, torch.bfloat16, seed=50 + T)
    g = _gpu(x, dO, dST, use_saved)
    ref = _oracle(x, dO, dST)
    for n in GRADS:
        assert_close(g[n], ref[n], TOL[torch.bfloat16], f"T={T} {n}")


def _edit(x, **fields):
    d = dict(x.__dict__)
    d.update(fields)
    return I.FwdInputs(**d)


@pytest.mark.parametrize("case", ["reset", "no_erase", "full_erase", "erase_range_2", "no_decay",
                                  "strong_decay", "decay_cliff", "one_hot_keys", "kda_gates", "slow_decay"])
def test_bf16_degenerate_cases(case):
    """The forward's degenerate inputs through the tensor-core backward. strong_decay and
    reset trip the decay-range guard, so their chunks take the pairwise-exponential path."""
    x, dO, dST = _case(1, 160, 2, 128, 128, torch.bfloat16, seed=60)
    la, b, k, w = x.log_alpha.clone(), x.b.clone(), x.k.clone(), x.w.clone()
    dt = torch.bfloat16
    if case == "reset":
        la[:, [3, 64, 100, 159]] = float("-inf")
    elif case == "no_erase":
        b.zero_()
    elif case == "full_erase":
        b.fill_(1.0)
    elif case == "erase_range_2":
        b = (b.float() * 2.0).to(dt)
    elif case == "no_decay":
        la.zero_()
    elif case == "strong_decay":
        la = la - 30.0
    elif case == "decay_cliff":
        prof = torch.zeros(64)
        prof[16:32] = -30.0 / 16
        prof[40:48] = -69.5 / 8
        la = prof.repeat(3)[:la.shape[1]][None, :, None, None].expand_as(la).contiguous()
    elif case == "one_hot_keys":
        k = torch.nn.functional.one_hot(torch.randint(0, 128, k.shape[:-1], generator=torch.Generator().manual_seed(0)),
                                        128).to(dt)
    elif case == "kda_gates":
        beta = torch.rand(b.shape[:-1], generator=torch.Generator().manual_seed(1))
        b = beta[..., None].expand_as(b).contiguous().to(dt)
        w = beta[..., None].expand_as(w).contiguous().to(dt)
    elif case == "slow_decay":
        la = -torch.nn.functional.softplus(torch.randn(la.shape, generator=torch.Generator().manual_seed(2)))
    x = _edit(x, log_alpha=la, b=b, k=k, w=w)
    for use_saved in (False, True):
        g = _gpu(x, dO, dST, use_saved)
        ref = _oracle(x, dO, dST)
        for n in GRADS:
            tol = TOL[torch.bfloat16]
            if case == "one_hot_keys" and n == "db":
                # With one-hot keys db = de (.) k is zero except where a key channel is hit
                # again within a few tokens (max|db| = 0.036 here against max|dk| = 21), and
                # there it is one near-orthogonal product dz_t . U_i (cosine 0.01) times a
                # decay factor: the 1e-3-level error that bf16 products leave in the forward's
                # states and in U becomes a few percent of it. A bf16-operand emulation of this
                # backward on the CPU gives 3.8e-2 on the same input.
                tol = 6e-2
            assert_close(g[n], ref[n], tol, f"{case} saved={use_saved} {n}")


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
