"""C-ABI checks that need no GPU: the library loads, exports every function
``include/gdr2.h`` declares, and rejects bad arguments on the host before any
launch (so no device work is enqueued)."""
import ctypes
import os
import re

import pytest

import gated_delta_rule_wy_b200 as g
from gated_delta_rule_wy_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from gated_delta_rule_wy_b200 import build

    build.build()
    return g.load_library()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "gdr2.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdr2_\w+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert declared_functions() == sorted(binding.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"libgdr2.so does not export {name}"


def test_abi_version(lib):
    assert lib.gdr2_abi_version() == 9


NULL11 = [None] * 11 + [ctypes.c_size_t(0), None]  # 11 tensors + workspace bytes + stream


@pytest.mark.parametrize("dims,dt,status", [
    ((1, 4, 1, 96, 64), 1, binding.GDR2_ERR_UNSUPPORTED),
    ((1, 4, 1, 64, 32), 1, binding.GDR2_ERR_UNSUPPORTED),
    ((-1, 4, 1, 64, 64), 1, binding.GDR2_ERR_INVALID_ARG),
    ((1, -4, 1, 64, 64), 1, binding.GDR2_ERR_INVALID_ARG),
    ((1, 4, 1, 0, 64), 1, binding.GDR2_ERR_INVALID_ARG),
    ((1, 4, 1, 64, 64), 7, binding.GDR2_ERR_INVALID_ARG),
    ((1, 4, 1, 64, 64), 1, binding.GDR2_ERR_INVALID_ARG),  # NULL q with tokens
])
def test_forward_rejects_bad_arguments(lib, dims, dt, status):
    assert lib.gdr2_forward(*dims, dt, *NULL11) == status
    assert lib.gdr2_last_error()


def test_forward_rejects_misaligned_pointer(lib):
    p = [ctypes.c_void_p(0x10000)] * 11
    p[2] = ctypes.c_void_p(0x10008)  # v
    assert lib.gdr2_forward(1, 4, 1, 64, 64, 1, *p, ctypes.c_size_t(0), None) == binding.GDR2_ERR_INVALID_ARG
    assert b"v is not 16-byte aligned" in lib.gdr2_last_error()


def test_decode_rejects_bad_arguments(lib):
    assert lib.gdr2_decode_step(2, 2, 128, 96, 1, *([None] * 9)) == binding.GDR2_ERR_UNSUPPORTED
    assert lib.gdr2_decode_step(2, 2, 128, 128, 1, *([None] * 9)) == binding.GDR2_ERR_INVALID_ARG
    # an empty batch is a no-op, even with NULL pointers
    assert lib.gdr2_decode_step(0, 16, 128, 128, 1, *([None] * 9)) == binding.GDR2_OK


def test_empty_problems_need_no_pointers(lib):
    assert lib.gdr2_forward(0, 128, 16, 128, 128, 1, *NULL11) == binding.GDR2_OK
    assert lib.gdr2_forward(4, 64, 0, 128, 128, 1, *NULL11) == binding.GDR2_OK


def test_backward_workspace_query_and_checks(lib):
    n = lib.gdr2_backward_workspace_bytes(2, 4096, 16, 128, 128, 1)
    # chunk states + one chunk of token states + deltas, per (batch, head)
    BH, NC, SS = 32, 64, 128 * 128 * 4
    assert n >= BH * NC * SS + BH * 65 * SS
    assert n % 256 == 0
    p = [ctypes.c_void_p(0x10000)] * 18  # 17 tensors + the workspace
    st = lib.gdr2_backward(2, 64, 16, 128, 128, 1, *p, ctypes.c_size_t(16), ctypes.c_void_p(0))
    assert st == binding.GDR2_ERR_INVALID_ARG and b"workspace" in lib.gdr2_last_error()
    assert lib.gdr2_backward_workspace_bytes(-1, 1, 1, 64, 64, 1) == 0


def test_varlen_forward_workspace_query_and_checks(lib):
    # slots and gamma vectors for at most H (ceil(T / 64) + N) tasks, then N + 2 ints
    n = lib.gdr2_forward_varlen_workspace_bytes(8, 1000, 16, 128, 128, 1)
    assert n >= 16 * (16 + 8) * (90112 + 512) + 10 * 4 and n % 256 == 0
    assert lib.gdr2_forward_varlen_workspace_bytes(8, 1000, 16, 128, 128, 0) == 0  # fp32: not supported
    p = ctypes.c_void_p(0x10000)
    args = [p] * 12 + [ctypes.c_size_t(1 << 30), ctypes.c_void_p(0)]
    assert lib.gdr2_forward_varlen(2, 64, 4, 128, 128, 0, 0, *args) == binding.GDR2_ERR_UNSUPPORTED
    assert lib.gdr2_forward_varlen(2, 64, 4, 64, 128, 1, 0, *args) == binding.GDR2_ERR_UNSUPPORTED
    assert lib.gdr2_forward_varlen(2, 64, 4, 128, 128, 1, 4, *args) == binding.GDR2_ERR_INVALID_ARG
    nul = [ctypes.c_void_p(0)] + [p] * 11 + [ctypes.c_size_t(1 << 30), ctypes.c_void_p(0)]
    st = lib.gdr2_forward_varlen(2, 64, 4, 128, 128, 1, 0, *nul)
    assert st == binding.GDR2_ERR_INVALID_ARG and b"cu_seqlens" in lib.gdr2_last_error()
    small = [p] * 12 + [ctypes.c_size_t(16), ctypes.c_void_p(0)]
    st = lib.gdr2_forward_varlen(2, 64, 4, 128, 128, 1, 0, *small)
    assert st == binding.GDR2_ERR_INVALID_ARG and b"workspace" in lib.gdr2_last_error()
    # no sequences or no heads: nothing to do, no pointer needed
    assert lib.gdr2_forward_varlen(0, 0, 4, 128, 128, 1, 0, *([ctypes.c_void_p(0)] * 12),
                                   ctypes.c_size_t(0), ctypes.c_void_p(0)) == binding.GDR2_OK


def test_gated_entry_points_check_the_gate_layout(lib):
    p = ctypes.c_void_p(0x10000)
    fwd = [p] * 11 + [ctypes.c_size_t(1 << 30), ctypes.c_void_p(0)]
    for bad in (-1, 4, 7):
        st = lib.gdr2_forward_gated(1, 64, 2, 128, 128, 1, bad, *fwd)
        assert st == binding.GDR2_ERR_INVALID_ARG and b"gates" in lib.gdr2_last_error()
        st = lib.gdr2_decode_step_gated(4, 2, 128, 128, 1, bad, *([p] * 9))
        assert st == binding.GDR2_ERR_INVALID_ARG and b"gates" in lib.gdr2_last_error()
    # a scalar gate needs element alignment only; a vector gate 16 bytes
    odd = ctypes.c_void_p(0x10002)
    args = [p, p, p, p, odd, odd] + [p] * 5 + [ctypes.c_size_t(0), ctypes.c_void_p(0)]
    st = lib.gdr2_forward_gated(1, 64, 2, 128, 128, 1, 0, *args)
    assert st == binding.GDR2_ERR_INVALID_ARG and b"16-byte" in lib.gdr2_last_error()
    st = lib.gdr2_forward_gated(1, 64, 2, 128, 128, 1, 3, *args)  # passes the gates, stops at the workspace
    assert st == binding.GDR2_ERR_INVALID_ARG and b"workspace" in lib.gdr2_last_error()
    odd1 = ctypes.c_void_p(0x10001)
    args = [p, p, p, p, odd1, p] + [p] * 5 + [ctypes.c_size_t(0), ctypes.c_void_p(0)]
    st = lib.gdr2_forward_gated(1, 64, 2, 128, 128, 1, 1, *args)
    assert st == binding.GDR2_ERR_INVALID_ARG and b"element size" in lib.gdr2_last_error()


def test_binding_validates_before_calling():
    import torch

    q = torch.zeros(1, 4, 1, 64)
    with pytest.raises(ValueError, match="CUDA"):
        g.gdr2_forward(q, q, q, q, q, q)


def test_noalloc_backward_rejects_oversized_problems_on_the_host(lib):
    """Too large for the built-in scratch array: UNSUPPORTED, nothing launched."""
    p = [ctypes.c_void_p(0x10000)] * 17 + [None]
    # 64 heads of d = 128 with saved states need ~270 MiB of scratch (> 64 MiB)
    st = lib.gdr2_backward_noalloc(4, 4096, 16, 128, 128, 1, *p)
    assert st == binding.GDR2_ERR_UNSUPPORTED
    assert b"GDR2_NOALLOC_SCRATCH_BYTES" in lib.gdr2_last_error()


def test_forward_workspace_query_and_check(lib):
    # bf16 at d = 128 runs on the tensor cores and needs the chunk workspace
    n = lib.gdr2_forward_workspace_bytes(4, 4096, 16, 128, 128, 1)
    ntasks = 4 * 16 * 64
    # per task a slot and its gamma, then the fused kernel's queue counter (16 bytes) and one
    # 4-byte flag per task, rounded up to 256 bytes
    assert n == ntasks * (90112 + 512) + (16 + 4 * ntasks + 255) // 256 * 256
    assert lib.gdr2_forward_workspace_bytes(4, 4096, 16, 128, 128, 0) == 0  # fp32: CUDA cores
    assert lib.gdr2_forward_workspace_bytes(4, 4096, 16, 64, 64, 1) == 0
    p = [ctypes.c_void_p(0x10000)] * 11  # 10 tensors + the workspace
    st = lib.gdr2_forward(1, 100, 1, 128, 128, 1, *p, ctypes.c_size_t(1024), None)
    assert st == binding.GDR2_ERR_INVALID_ARG and b"workspace" in lib.gdr2_last_error()


def _ex_args(out_gate, norm_weight, eps, cu=None, ws_bytes=1 << 30):
    p = ctypes.c_void_p(0x10000)
    return ([cu] + [p] * 6 + [None] + [out_gate, norm_weight, ctypes.c_float(eps)] + [p, None, None, p] +
            [ctypes.c_size_t(ws_bytes), ctypes.c_void_p(0)])


def test_forward_ex_checks_the_epilogue_on_the_host(lib):
    p, odd = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10008)
    # the epilogue runs on the tensor-core path only: fp32 or d = 64 are UNSUPPORTED
    st = lib.gdr2_forward_ex(1, 64, 2, 128, 128, 0, 0, *_ex_args(None, p, 1e-6))
    assert st == binding.GDR2_ERR_UNSUPPORTED and b"norm" in lib.gdr2_last_error()
    st = lib.gdr2_forward_ex(1, 64, 2, 64, 64, 1, 0, *_ex_args(p, None, 1e-6))
    assert st == binding.GDR2_ERR_UNSUPPORTED
    # the gate has o's layout: 16-byte aligned; the weight 4-byte aligned; eps finite, >= 0
    st = lib.gdr2_forward_ex(1, 64, 2, 128, 128, 1, 0, *_ex_args(odd, None, 1e-6))
    assert st == binding.GDR2_ERR_INVALID_ARG and b"out_gate" in lib.gdr2_last_error()
    st = lib.gdr2_forward_ex(1, 64, 2, 128, 128, 1, 0, *_ex_args(None, ctypes.c_void_p(0x10002), 1e-6))
    assert st == binding.GDR2_ERR_INVALID_ARG and b"norm_weight" in lib.gdr2_last_error()
    for eps in (-1e-6, float("nan"), float("inf")):
        st = lib.gdr2_forward_ex(1, 64, 2, 128, 128, 1, 0, *_ex_args(None, p, eps))
        assert st == binding.GDR2_ERR_INVALID_ARG and b"norm_eps" in lib.gdr2_last_error()
    # eps is not looked at without a norm; valid arguments stop at the workspace check here
    st = lib.gdr2_forward_ex(1, 64, 2, 128, 128, 1, 0, *_ex_args(p, None, -1.0, ws_bytes=16))
    assert st == binding.GDR2_ERR_INVALID_ARG and b"workspace" in lib.gdr2_last_error()
    # packed: the varlen workspace is the one asked for
    cu = ctypes.c_void_p(0x20000)
    need = lib.gdr2_forward_varlen_workspace_bytes(3, 64, 2, 128, 128, 1)
    st = lib.gdr2_forward_ex(3, 64, 2, 128, 128, 1, 0, *_ex_args(p, p, 1e-6, cu=cu, ws_bytes=need - 256))
    assert st == binding.GDR2_ERR_INVALID_ARG and b"workspace" in lib.gdr2_last_error()
    st = lib.gdr2_forward_ex(3, 64, 2, 128, 128, 0, 0, *_ex_args(None, None, 0.0, cu=cu))
    assert st == binding.GDR2_ERR_UNSUPPORTED and b"packed" in lib.gdr2_last_error()


def test_prologue_entry_points_check_on_the_host(lib):
    p, q = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x20000)
    f = ctypes.c_float

    def conv(N=2, T=8, H=2, d=128, dt=1, W=4, l2=1, eps=1e-6, cu=None, x=p, wgt=p, sin=None, sout=None, y=q):
        return lib.gdr2_short_conv_silu(N, T, H, d, dt, W, l2, f(eps), cu, x, wgt, sin, sout, y, None)

    assert conv(W=5) == binding.GDR2_ERR_UNSUPPORTED and b"width" in lib.gdr2_last_error()
    assert conv(W=0) == binding.GDR2_ERR_UNSUPPORTED
    assert conv(d=96) == binding.GDR2_ERR_UNSUPPORTED
    assert conv(N=-1) == binding.GDR2_ERR_INVALID_ARG
    assert conv(l2=2) == binding.GDR2_ERR_INVALID_ARG
    assert conv(eps=-1.0) == binding.GDR2_ERR_INVALID_ARG and b"l2_eps" in lib.gdr2_last_error()
    assert conv(y=p) == binding.GDR2_ERR_INVALID_ARG and b"y must not be x" in lib.gdr2_last_error()
    assert conv(x=ctypes.c_void_p(0x10008)) == binding.GDR2_ERR_INVALID_ARG
    assert conv(wgt=None) == binding.GDR2_ERR_INVALID_ARG and b"weight" in lib.gdr2_last_error()
    s = ctypes.c_void_p(0x30000)
    st = conv(sin=s, sout=s)  # in place needs T = 1 without cu_seqlens
    assert st == binding.GDR2_ERR_INVALID_ARG and b"state_in" in lib.gdr2_last_error()
    st = conv(T=1, sin=s, sout=s, cu=ctypes.c_void_p(0x40000))
    assert st == binding.GDR2_ERR_INVALID_ARG
    assert conv(cu=ctypes.c_void_p(0x40002)) == binding.GDR2_ERR_INVALID_ARG  # cu_seqlens alignment
    assert conv(N=0, x=None, wgt=None, y=None) == binding.GDR2_OK  # nothing to do
    assert conv(H=0, x=None, wgt=None, y=None) == binding.GDR2_OK

    def act(dt=1, na=16, a=p, la=q, nb=0, b=None, bo=None, nw=0, w=None, wo=None):
        return lib.gdr2_gate_activations(dt, na, a, la, nb, b, bo, nw, w, wo, None)

    assert act(dt=5) == binding.GDR2_ERR_INVALID_ARG
    assert act(na=-1) == binding.GDR2_ERR_INVALID_ARG
    assert act(la=None) == binding.GDR2_ERR_INVALID_ARG and b"both or neither" in lib.gdr2_last_error()
    assert act(a=ctypes.c_void_p(0x10004)) == binding.GDR2_ERR_INVALID_ARG and b"aligned" in lib.gdr2_last_error()
    assert act(la=p) == binding.GDR2_ERR_INVALID_ARG  # bf16 a cannot become fp32 log_alpha in place
    assert act(na=0, a=None, la=None) == binding.GDR2_OK


def test_segment_states_checks_on_the_host(lib):
    p = ctypes.c_void_p(0x10000)
    assert lib.gdr2_segment_states(2, 3, 2, 96, 128, p, p, None, p, None, None) == binding.GDR2_ERR_UNSUPPORTED
    assert lib.gdr2_segment_states(-1, 3, 2, 128, 128, p, p, None, p, None, None) == binding.GDR2_ERR_INVALID_ARG
    st = lib.gdr2_segment_states(2, 3, 2, 128, 128, None, p, None, p, None, None)
    assert st == binding.GDR2_ERR_INVALID_ARG and b"A is NULL" in lib.gdr2_last_error()
    st = lib.gdr2_segment_states(2, 3, 2, 128, 128, p, p, ctypes.c_void_p(0x10004), p, None, None)
    assert st == binding.GDR2_ERR_INVALID_ARG and b"S0" in lib.gdr2_last_error()
    assert lib.gdr2_segment_states(0, 3, 2, 128, 128, None, None, None, None, None, None) == binding.GDR2_OK


def test_new_binding_functions_validate_before_calling():
    import torch

    x = torch.zeros(1, 8, 2, 64)
    with pytest.raises(ValueError, match="CUDA"):
        g.gdr2_short_conv_silu(x, torch.zeros(128, 4))
    with pytest.raises(ValueError, match="multiple of segments"):
        g.gdr2_forward_segmented(x, x, x, x, x, x, segments=3)
    with pytest.raises(ValueError, match="CUDA"):
        g.gdr2_segment_states(torch.zeros(1, 2, 2, 64, 64), torch.zeros(1, 2, 2, 64, 64))
    with pytest.raises(ValueError, match="CUDA"):
        g.gdr2_gate_activations(torch.zeros(16))


def test_binding_rejects_tensors_on_several_devices():
    """Every tensor of a call and its stream must be on one device: the library launches on
    the current device, so a tensor elsewhere would reach a kernel as a foreign pointer."""
    import torch

    from gated_delta_rule_wy_b200.binding import _device_of

    host, meta = torch.zeros(1, 4, 1, 64), torch.zeros(1, 4, 1, 64, device="meta")
    with pytest.raises(ValueError, match="one CUDA device"):
        _device_of([host, meta])
    with pytest.raises(ValueError, match="one CUDA device"):
        g.gdr2_forward(host, host, meta, host, host, host)
    with pytest.raises(ValueError, match="one CUDA device"):
        g.gdr2_backward(host, host, host, host, host, host, meta)
    assert _device_of([host, host]) == torch.device("cpu")
