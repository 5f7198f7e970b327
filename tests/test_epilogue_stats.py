"""The parity statistics of the output epilogue, pinned on the CPU.

A correct epilogue applied to a mixer output carrying an error of the size the bf16
path shows (about 5e-3 of max|o|) passes; each plausible mistake in the epilogue,
planted in the oracle's epilogue here, fails at the bound the GPU tests use:
the implied-mixer-error statistic on the full path, the plain max-relative error in
the well-conditioned case (k = 0, no decay, weights ~ N(0, 1)).
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from oracle.block import output_norm_gate, silu
from gated_delta_rule_wy_b200 import inputs as I
from parity import TOL, epilogue_err, rel_err

TOLB = TOL[torch.bfloat16]


def _bf16(a):
    return torch.tensor(a).to(torch.bfloat16).double().numpy()


def _noisy(o, seed):
    rng = np.random.default_rng(seed)
    return o * (1 + 4e-3 * rng.standard_normal(o.shape)) + 1e-3 * np.abs(o).max() * rng.standard_normal(o.shape)


@pytest.fixture(scope="module")
def full_path():
    x = I.make_forward_inputs(B=1, H=3, T=160, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=91,
                              with_S0=True)
    g, w = I.make_epilogue_inputs((1, 160, 3, 128), 128, seed=92)
    n = x.as_numpy64()
    o_ref, _ = oracle.forward(n["q"], n["k"], n["v"], n["log_alpha"], n["b"], n["w"], S0=n["S0"])
    return o_ref, g.double().numpy(), w.double().numpy()


FULL_MUTANTS = {
    "sigmoid instead of silu": lambda o, g, w, e: output_norm_gate(o, None, w, e) / (1 + np.exp(-g)),
    "sum instead of mean": lambda o, g, w, e: o / np.sqrt((o * o).sum(-1, keepdims=True) + e) * w * silu(g),
    "gate of the previous token": lambda o, g, w, e: output_norm_gate(o, np.roll(g, 1, axis=1), w, e),
    "gate channels shifted": lambda o, g, w, e: output_norm_gate(o, np.roll(g, 1, axis=-1), w, e),
    "rms over heads": lambda o, g, w, e: o / np.sqrt((o * o).mean(-2, keepdims=True) + e) * w * silu(g),
    "weight reversed": lambda o, g, w, e: output_norm_gate(o, g, w[::-1], e),
}


def test_full_path_statistic_passes_the_correct_epilogue(full_path):
    o_ref, g, w = full_path
    y_ref = output_norm_gate(o_ref, g, w, 1e-6)
    y = _bf16(output_norm_gate(_noisy(o_ref, 1), g, w, 1e-6))
    assert epilogue_err(y, y_ref, o_ref, g, w, 1e-6) < TOLB / 4
    assert epilogue_err(y_ref, y_ref, o_ref, g, w, 1e-6) == 0.0
    # gate only, norm only
    assert epilogue_err(_bf16(_noisy(o_ref, 2) * silu(g)), o_ref * silu(g), o_ref, g, None, 1e-6) < TOLB / 4
    yn = output_norm_gate(o_ref, None, w, 1e-6)
    assert epilogue_err(_bf16(output_norm_gate(_noisy(o_ref, 3), None, w, 1e-6)), yn, o_ref, None, w, 1e-6) < TOLB / 4


@pytest.mark.parametrize("name", list(FULL_MUTANTS))
def test_full_path_statistic_rejects_a_wrong_epilogue(full_path, name):
    o_ref, g, w = full_path
    y_ref = output_norm_gate(o_ref, g, w, 1e-6)
    y = _bf16(FULL_MUTANTS[name](_noisy(o_ref, 1), g, w, 1e-6))
    assert epilogue_err(y, y_ref, o_ref, g, w, 1e-6) > TOLB, name


@pytest.fixture(scope="module")
def well_conditioned():
    x = I.make_forward_inputs(B=1, H=3, T=96, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=101,
                              with_S0=True)
    x = dataclasses.replace(x, k=torch.zeros_like(x.k), log_alpha=torch.zeros_like(x.log_alpha))
    g, _ = I.make_epilogue_inputs((1, 96, 3, 128), 128, seed=102)
    w = torch.randn(128, generator=torch.Generator().manual_seed(103)).double().numpy()
    n = x.as_numpy64()
    o_ref, _ = oracle.forward(n["q"], n["k"], n["v"], n["log_alpha"], n["b"], n["w"], S0=n["S0"])
    # k = 0 and alpha = 1: the state never moves, o_t = S0^T q_t
    assert np.allclose(o_ref[0], np.einsum("hcj,thc->thj", n["S0"][0], n["q"][0]), rtol=0, atol=1e-12)
    r = np.sqrt((o_ref ** 2).mean(-1))
    assert r.min() > 0.5 * r.max()  # every token's output of similar size
    return o_ref, g.double().numpy(), w


WC_MUTANTS = {
    "no weight": lambda o, g, w, e: output_norm_gate(o, g, np.ones_like(w), e),
    "weight reversed": lambda o, g, w, e: output_norm_gate(o, g, w[::-1], e),
    "eps ignored": lambda o, g, w, e: output_norm_gate(o, g, w, 0.0),
    "eps outside the root": lambda o, g, w, e: o / (np.sqrt((o * o).mean(-1, keepdims=True)) + e) * w * silu(g),
    "rms of half the channels": lambda o, g, w, e: o / np.sqrt((o[..., :64] ** 2).mean(-1, keepdims=True) + e)
    * w * silu(g),
    "sigmoid instead of silu": lambda o, g, w, e: output_norm_gate(o, None, w, e) / (1 + np.exp(-g)),
}


def test_well_conditioned_bound_passes_the_correct_epilogue(well_conditioned):
    o_ref, g, w = well_conditioned
    for eps in (1e-6, 1e-2):
        y_ref = output_norm_gate(o_ref, g, w, eps)
        assert rel_err(_bf16(output_norm_gate(_noisy(o_ref, 4), g, w, eps)), y_ref) < TOLB / 2


@pytest.mark.parametrize("name", list(WC_MUTANTS))
def test_well_conditioned_bound_rejects_a_wrong_epilogue(well_conditioned, name):
    o_ref, g, w = well_conditioned
    y_ref = output_norm_gate(o_ref, g, w, 1e-2)
    y = _bf16(WC_MUTANTS[name](_noisy(o_ref, 4), g, w, 1e-2))
    assert rel_err(y, y_ref) > TOLB, name
