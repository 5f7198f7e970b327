"""The fused forward kernel against the two-kernel forward it replaces (needs a B200).

Where B H leaves at least 32 SMs to the chunk tasks, a dense bf16 forward runs as one cooperative
launch: every CTA takes chunk tasks from a queue in chunk-major order, and CTA b < B H then runs
the scan of (sequence, head) b, reading each chunk's workspace slot once its flag is set. Every
product is the one the two-kernel forward (all chunk tasks, then one scan kernel) computes, in
the same order, so the outputs must be the same bits; gdr2_debug_forward_unfused selects the two
kernels for the comparison. Parity of either against the oracle is covered by the forward tests.
"""
import pytest
import torch

from gated_delta_rule_wy_b200 import binding, gdr2_forward, gdr2_sync_status
from gated_delta_rule_wy_b200 import inputs as I

pytestmark = pytest.mark.gpu

CASES = [
    # 4 chunks with a ragged tail: both scan CTAs leave the queue after their first task
    dict(B=1, H=2, T=200, seed=81, with_S0=True),
    dict(B=2, H=3, T=1000, seed=82, with_S0=False, decay_shift=2.0),
    # the 1.3B layer: 64 scans, the switch in the queue's last fifth
    dict(B=4, H=16, T=4096, seed=83, with_S0=False),
    # long sequences: 32 scans of 512 chunks, switching about halfway through the queue
    dict(B=2, H=16, T=32768, seed=84, with_S0=True),
]


# edges: B H at the fusion threshold of a 148-SM B200 (116 scans beside 32 queue CTAs), one
# chunk, one token, one (sequence, head), a chunk count that the scans' switch index hits early
CASES += [
    dict(B=4, H=29, T=130, seed=90, with_S0=True),
    dict(B=3, H=5, T=64, seed=91, with_S0=True),
    dict(B=2, H=3, T=1, seed=92, with_S0=True),
    dict(B=1, H=1, T=777, seed=93, with_S0=True, decay_shift=2.0),
]


@pytest.mark.parametrize("c", CASES, ids=lambda c: f"B{c['B']}_H{c['H']}_T{c['T']}")
def test_fused_forward_is_bitwise_the_two_kernel_forward(c):
    lib = binding.load_library()
    x = I.make_forward_inputs(B=c["B"], H=c["H"], T=c["T"], dk=128, dv=128, dtype=torch.bfloat16,
                              decay_shift=c.get("decay_shift", 0.0), seed=c["seed"],
                              with_S0=c["with_S0"]).to("cuda")
    o1, S1, _ = gdr2_forward(x.q, x.k, x.v, x.log_alpha, x.b, x.w, x.S0)
    gdr2_sync_status()
    lib.gdr2_debug_forward_unfused(1)
    try:
        o2, S2, _ = gdr2_forward(x.q, x.k, x.v, x.log_alpha, x.b, x.w, x.S0)
        gdr2_sync_status()
    finally:
        lib.gdr2_debug_forward_unfused(0)
    assert torch.isfinite(o1.float()).all()
    assert torch.equal(o1, o2), f"o differs in {(o1 != o2).sum().item()} elements"
    assert torch.equal(S1, S2), f"S_T differs in {(S1 != S2).sum().item()} elements"


def test_fused_forward_reused_workspace_and_back_to_back_calls():
    # the queue and flags are cleared by every call: a workspace holding a finished call's flags
    # (all set) must not let the next call's scans read slots before they are written
    lib = binding.load_library()
    x = I.make_forward_inputs(B=2, H=8, T=2048, dk=128, dv=128, dtype=torch.bfloat16, seed=85).to("cuda")
    from gated_delta_rule_wy_b200 import gdr2_forward_workspace_bytes
    ws = torch.empty(gdr2_forward_workspace_bytes(2, 2048, 8, 128, 128, torch.bfloat16), dtype=torch.uint8,
                     device="cuda")
    lib.gdr2_debug_forward_unfused(1)
    try:
        ref, _, _ = gdr2_forward(x.q, x.k, x.v, x.log_alpha, x.b, x.w, None, workspace=ws)
        gdr2_sync_status()
    finally:
        lib.gdr2_debug_forward_unfused(0)
    outs = [gdr2_forward(x.q, x.k, x.v, x.log_alpha, x.b, x.w, None, workspace=ws)[0] for _ in range(4)]
    gdr2_sync_status()
    for o in outs:
        assert torch.equal(o, ref)


@pytest.mark.parametrize("scalar", ["b", "w", "bw"])
def test_fused_forward_with_scalar_gates_is_bitwise_the_two_kernel_forward(scalar):
    # scalar gates take the general chunk body, fused the same way
    lib = binding.load_library()
    B, H, T = 2, 8, 3000
    x = I.make_forward_inputs(B=B, H=H, T=T, dk=128, dv=128, dtype=torch.bfloat16, seed=86, with_S0=True).to("cuda")
    b = x.b[..., 0].contiguous() if "b" in scalar else x.b
    w = x.w[..., 0].contiguous() if "w" in scalar else x.w
    o1, S1, _ = gdr2_forward(x.q, x.k, x.v, x.log_alpha, b, w, x.S0)
    gdr2_sync_status()
    lib.gdr2_debug_forward_unfused(1)
    try:
        o2, S2, _ = gdr2_forward(x.q, x.k, x.v, x.log_alpha, b, w, x.S0)
        gdr2_sync_status()
    finally:
        lib.gdr2_debug_forward_unfused(0)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


BWD_CASES = [
    dict(B=1, H=2, T=200, seed=87, with_S0=True, dS_T=True),   # ragged tail, both scans switch at once
    dict(B=2, H=16, T=4096, seed=88, with_S0=False, dS_T=False),  # the benchmarked backward
    dict(B=2, H=4, T=1500, seed=89, with_S0=True, dS_T=True, scalar="bw"),
]


@pytest.mark.parametrize("c", BWD_CASES, ids=lambda c: f"B{c['B']}_H{c['H']}_T{c['T']}{'_' + c.get('scalar', '')}")
def test_fused_backward_front_is_bitwise_the_two_launch_front(c):
    # with saved states the backward's chunk tasks and reverse scans run as one cooperative launch
    # (chunk-major from the last chunk); every gradient must be the same bits as with the two
    # launches it replaces
    from gated_delta_rule_wy_b200 import gdr2_backward
    lib = binding.load_library()
    x = I.make_forward_inputs(B=c["B"], H=c["H"], T=c["T"], dk=128, dv=128, dtype=torch.bfloat16, seed=c["seed"],
                              with_S0=c["with_S0"]).to("cuda")
    b = x.b[..., 0].contiguous() if "b" in c.get("scalar", "") else x.b
    w = x.w[..., 0].contiguous() if "w" in c.get("scalar", "") else x.w
    dO = I.make_upstream_grad(c["B"], c["T"], c["H"], 128, c["seed"], dtype=torch.bfloat16).cuda()
    dS_T = (torch.randn((c["B"], c["H"], 128, 128), generator=torch.Generator().manual_seed(c["seed"])) * 0.1).cuda() \
        if c["dS_T"] else None
    _, _, saved = gdr2_forward(x.q, x.k, x.v, x.log_alpha, b, w, x.S0, save_states=True)
    g1 = gdr2_backward(x.q, x.k, x.v, x.log_alpha, b, w, dO, x.S0, dS_T, saved)
    gdr2_sync_status()
    lib.gdr2_debug_forward_unfused(1)
    try:
        g2 = gdr2_backward(x.q, x.k, x.v, x.log_alpha, b, w, dO, x.S0, dS_T, saved)
        gdr2_sync_status()
    finally:
        lib.gdr2_debug_forward_unfused(0)
    for name in g1:
        if g1[name] is None:
            assert g2[name] is None
            continue
        assert torch.isfinite(g1[name].float()).all(), name
        assert torch.equal(g1[name], g2[name]), f"{name} differs in {(g1[name] != g2[name]).sum().item()} elements"


@pytest.mark.parametrize("shape", [(1, 2, 200), (2, 16, 4096)], ids=["B1_H2_T200", "B2_H16_T4096"])
def test_fused_forward_with_saved_states_and_the_recomputing_backward(shape):
    # the forward's saved chunk states, and the backward without them (which recomputes them in
    # the fused forward launch, keeping T and W for its chunk kernels), against the two kernels
    from gated_delta_rule_wy_b200 import gdr2_backward
    lib = binding.load_library()
    B, H, T = shape
    x = I.make_forward_inputs(B=B, H=H, T=T, dk=128, dv=128, dtype=torch.bfloat16, seed=94, with_S0=True).to("cuda")
    dO = I.make_upstream_grad(B, T, H, 128, 94, dtype=torch.bfloat16).cuda()
    dS_T = (torch.randn((B, H, 128, 128), generator=torch.Generator().manual_seed(95)) * 0.1).cuda()
    runs = []
    for unfused in (0, 1):
        lib.gdr2_debug_forward_unfused(unfused)
        try:
            o, S, saved = gdr2_forward(x.q, x.k, x.v, x.log_alpha, x.b, x.w, x.S0, save_states=True)
            g = gdr2_backward(x.q, x.k, x.v, x.log_alpha, x.b, x.w, dO, x.S0, dS_T, None)
            gdr2_sync_status()
        finally:
            lib.gdr2_debug_forward_unfused(0)
        runs.append((o, S, saved, g))
    (o1, S1, sv1, g1), (o2, S2, sv2, g2) = runs
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    assert torch.equal(sv1, sv2), "saved states differ"
    for name in g1:
        if g1[name] is not None:
            assert torch.equal(g1[name], g2[name]), name
