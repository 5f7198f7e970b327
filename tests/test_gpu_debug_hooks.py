"""Device code that normal inputs never reach, through the C ABI's test hooks (needs a B200).

gdr2_debug_force_timeout makes the forward's chunk work (also inside the fused forward and
the backward's fused front) give up a 1 us bounded wait before it issues anything: the
give-up path (TMEM freed, status word set, kernel returns) then runs, and the library must
report GDR2_ERR_TIMEOUT and stay usable. gdr2_debug_recip
evaluates the reciprocal the kernels use on the FMA pipe.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_wy_b200 import binding, gdr2_forward, gdr2_sync_status
from gated_delta_rule_wy_b200 import inputs as I
from parity import TOL, assert_close

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_the_library_stays_usable():
    lib = binding.load_library()
    x = I.make_forward_inputs(B=1, H=2, T=200, dk=128, dv=128, dtype=torch.bfloat16, decay_shift=2.0, seed=71,
                              with_S0=True)
    d = x.to("cuda")
    gdr2_sync_status()  # a clean status word to start from
    lib.gdr2_debug_force_timeout(1)
    try:
        gdr2_forward(d.q, d.k, d.v, d.log_alpha, d.b, d.w, d.S0)
        with pytest.raises(binding.GDR2Error, match="TIMEOUT"):
            gdr2_sync_status()
    finally:
        lib.gdr2_debug_force_timeout(0)
    gdr2_sync_status()  # the word was cleared by the report
    o, S_T, _ = gdr2_forward(d.q, d.k, d.v, d.log_alpha, d.b, d.w, d.S0)
    gdr2_sync_status()
    n = x.as_numpy64()
    o_ref, S_ref = oracle.forward(n["q"], n["k"], n["v"], n["log_alpha"], n["b"], n["w"], S0=n["S0"])
    assert_close(o, o_ref, TOL[torch.bfloat16], "o after the give-up")
    assert_close(S_T, S_ref, TOL[torch.bfloat16], "S_T after the give-up")


def test_backward_gives_up_in_its_fused_front_and_the_library_stays_usable():
    # with saved states the backward's chunk tasks and reverse scans are one cooperative launch;
    # its chunk role takes the same give-up path, and the scans that wait on it never start
    from gated_delta_rule_wy_b200 import gdr2_backward
    lib = binding.load_library()
    x = I.make_forward_inputs(B=1, H=2, T=300, dk=128, dv=128, dtype=torch.bfloat16, seed=73, with_S0=True)
    d = x.to("cuda")
    dO = I.make_upstream_grad(1, 300, 2, 128, 73, dtype=torch.bfloat16).cuda()
    _, _, saved = gdr2_forward(d.q, d.k, d.v, d.log_alpha, d.b, d.w, d.S0, save_states=True)
    ref = gdr2_backward(d.q, d.k, d.v, d.log_alpha, d.b, d.w, dO, d.S0, None, saved)
    gdr2_sync_status()
    lib.gdr2_debug_force_timeout(1)
    try:
        gdr2_backward(d.q, d.k, d.v, d.log_alpha, d.b, d.w, dO, d.S0, None, saved)
        with pytest.raises(binding.GDR2Error, match="TIMEOUT"):
            gdr2_sync_status()
    finally:
        lib.gdr2_debug_force_timeout(0)
    gdr2_sync_status()
    again = gdr2_backward(d.q, d.k, d.v, d.log_alpha, d.b, d.w, dO, d.S0, None, saved)
    gdr2_sync_status()
    for name, g in ref.items():
        if g is not None:
            assert torch.equal(again[name], g), name


def test_device_reciprocal_against_division():
    lib = binding.load_library()
    rng = np.random.default_rng(72)
    # log-uniform over the callers' range and beyond (2^-126 .. 2^124), binade edges included
    e = rng.uniform(-126.0, 124.0, 1 << 20)
    x = np.concatenate([np.exp2(e), np.exp2(np.arange(-126, 125, dtype=np.float64)),
                        np.nextafter(np.exp2(np.arange(-125, 125, dtype=np.float64)), 0)]).astype(np.float32)
    xd = torch.from_numpy(x).cuda()
    yd = torch.empty_like(xd)
    st = lib.gdr2_debug_recip(ctypes.c_void_p(xd.data_ptr()), ctypes.c_void_p(yd.data_ptr()), x.size,
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == binding.GDR2_OK
    torch.cuda.synchronize()
    rel = yd.cpu().double().numpy() * x.astype(np.float64) - 1.0
    assert np.max(np.abs(rel)) <= 6.6e-6
