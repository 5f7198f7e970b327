"""ctypes binding of libgdr2.so: the C ABI in ``include/gdr2.h`` with torch tensors.

Argument marshalling only. Every function here checks shapes, dtypes and
devices, allocates output tensors with PyTorch (device memory is the one
thing torch provides), passes raw device pointers and the current CUDA stream
to the library, and turns a non-OK status into ``GDR2Error``. There is no
fallback: if ``libgdr2.so`` is missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import functools
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdr2.so")

GDR2_OK, GDR2_ERR_INVALID_ARG, GDR2_ERR_UNSUPPORTED, GDR2_ERR_CUDA, GDR2_ERR_TIMEOUT = range(5)
GDR2_F32, GDR2_BF16 = 0, 1
CHUNK = 64
_STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CUDA", 4: "TIMEOUT"}

# Every symbol include/gdr2.h declares (the ABI tests check the exports).
EXPORTED_SYMBOLS = ("gdr2_abi_version", "gdr2_last_error", "gdr2_forward_workspace_bytes", "gdr2_forward",
                    "gdr2_forward_gated", "gdr2_forward_varlen_workspace_bytes", "gdr2_forward_varlen",
                    "gdr2_forward_ex", "gdr2_short_conv_silu", "gdr2_gate_activations", "gdr2_segment_states",
                    "gdr2_decode_step", "gdr2_decode_step_gated",
                    "gdr2_backward_workspace_bytes", "gdr2_backward", "gdr2_backward_gated", "gdr2_backward_noalloc",
                    "gdr2_sync_status", "gdr2_debug_force_timeout", "gdr2_debug_recip",
                    "gdr2_debug_forward_unfused")
NOALLOC_SCRATCH_BYTES = 64 << 20  # GDR2_NOALLOC_SCRATCH_BYTES


class GDR2Error(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"GDR2 {_STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_lock = threading.Lock()
_lib = None


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load libgdr2.so once and declare the signatures of include/gdr2.h."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"{p} is missing: build it with `python -m gated_delta_rule_wy_b200.build` "
                               "(there is no CPU fallback)")
        lib = ctypes.CDLL(p)
        I, P, Z = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
        lib.gdr2_abi_version.restype = I
        lib.gdr2_abi_version.argtypes = []
        lib.gdr2_last_error.restype = ctypes.c_char_p
        lib.gdr2_last_error.argtypes = []
        lib.gdr2_forward_workspace_bytes.restype = Z
        lib.gdr2_forward_workspace_bytes.argtypes = [I, I, I, I, I, I]
        lib.gdr2_forward.restype = I
        lib.gdr2_forward.argtypes = [I, I, I, I, I, I] + [P] * 11 + [Z, P]
        lib.gdr2_decode_step.restype = I
        lib.gdr2_forward_varlen_workspace_bytes.restype = Z
        lib.gdr2_forward_varlen_workspace_bytes.argtypes = [I, I, I, I, I, I]
        lib.gdr2_forward_varlen.restype = I
        lib.gdr2_forward_varlen.argtypes = [I, I, I, I, I, I, I] + [P] * 12 + [Z, P]
        lib.gdr2_forward_ex.restype = I
        lib.gdr2_forward_ex.argtypes = [I, I, I, I, I, I, I] + [P] * 8 + [P, P, ctypes.c_float] + [P] * 4 + [Z, P]
        lib.gdr2_short_conv_silu.restype = I
        lib.gdr2_short_conv_silu.argtypes = [I] * 7 + [ctypes.c_float] + [P] * 7
        lib.gdr2_gate_activations.restype = I
        lib.gdr2_gate_activations.argtypes = [I] + [ctypes.c_longlong, P, P] * 3 + [P]
        lib.gdr2_segment_states.restype = I
        lib.gdr2_segment_states.argtypes = [I] * 5 + [P] * 6
        lib.gdr2_forward_gated.restype = I
        lib.gdr2_forward_gated.argtypes = [I, I, I, I, I, I, I] + [P] * 11 + [Z, P]
        lib.gdr2_decode_step_gated.restype = I
        lib.gdr2_decode_step_gated.argtypes = [I, I, I, I, I, I] + [P] * 9
        lib.gdr2_decode_step.argtypes = [I, I, I, I, I] + [P] * 9
        lib.gdr2_backward_workspace_bytes.restype = Z
        lib.gdr2_backward_workspace_bytes.argtypes = [I, I, I, I, I, I]
        lib.gdr2_backward.restype = I
        lib.gdr2_backward.argtypes = [I, I, I, I, I, I] + [P] * 18 + [Z, P]
        lib.gdr2_backward_gated.restype = I
        lib.gdr2_backward_gated.argtypes = [I, I, I, I, I, I, I] + [P] * 18 + [Z, P]
        lib.gdr2_backward_noalloc.restype = I
        lib.gdr2_backward_noalloc.argtypes = [I, I, I, I, I, I] + [P] * 18
        lib.gdr2_sync_status.restype = I
        lib.gdr2_sync_status.argtypes = [P]
        lib.gdr2_debug_force_timeout.restype = None
        lib.gdr2_debug_force_timeout.argtypes = [I]
        lib.gdr2_debug_forward_unfused.restype = None
        lib.gdr2_debug_forward_unfused.argtypes = [I]
        lib.gdr2_debug_recip.restype = I
        lib.gdr2_debug_recip.argtypes = [P, P, ctypes.c_longlong, P]
        _lib = lib
        return lib


def _tensors_in(args, kwargs):
    for a in list(args) + list(kwargs.values()):
        if isinstance(a, torch.Tensor):
            yield a
        elif isinstance(a, (list, tuple)):
            yield from (x for x in a if isinstance(x, torch.Tensor))


def _device_of(tensors):
    """The one device the tensors live on (None without tensors); raises if they span several."""
    devs = {t.device for t in tensors}
    if len(devs) > 1:
        names = ", ".join(sorted(str(d) for d in devs))
        raise ValueError(f"all tensors of a call must be on one CUDA device; got {names}")
    return next(iter(devs)) if devs else None


def _one_device(fn):
    """Run a library call on the device that holds its tensors.

    The library launches on the current CUDA device and stream, so tensors on another
    device would reach kernels as foreign pointers: the call is made under that device
    (its current stream unless one is given), after checking that every tensor argument
    and the stream share it.
    """
    @functools.wraps(fn)
    def call(*args, **kwargs):
        dev = _device_of(_tensors_in(args, kwargs))
        if dev is None or dev.type != "cuda":
            return fn(*args, **kwargs)  # the argument checks reject host tensors
        stream = kwargs.get("stream")
        if stream is not None and stream.device != dev:
            raise ValueError(f"the stream is on {stream.device}, the tensors on {dev}: one CUDA device per call")
        with torch.cuda.device(dev):
            return fn(*args, **kwargs)
    return call


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return GDR2_F32
    if t.dtype == torch.bfloat16:
        return GDR2_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _check(t, name, shape, dtype):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")


GATE_SCALAR_B, GATE_SCALAR_W = 1, 2  # GDR2_GATE_* of include/gdr2.h


def _gates(b, w, lead):
    """Gate layout bits from the shapes: a gate shaped `lead` (no channel dim) is a scalar."""
    g = 0
    if tuple(b.shape) == tuple(lead):
        g |= GATE_SCALAR_B
    if tuple(w.shape) == tuple(lead):
        g |= GATE_SCALAR_W
    return g


def _epilogue(out_gate, norm_weight, o_shape, dv, dt, dev):
    """Checks the output gate and norm weight; True when either is given."""
    if out_gate is not None:
        _check(out_gate, "out_gate", o_shape, dt)
        if out_gate.device != dev:
            raise ValueError("out_gate must be on the inputs' device")
    if norm_weight is not None:
        _check(norm_weight, "norm_weight", (dv,), torch.float32)
        if norm_weight.device != dev:
            raise ValueError("norm_weight must be on the inputs' device")
    return out_gate is not None or norm_weight is not None


def _raise(lib, st):
    if st != GDR2_OK:
        raise GDR2Error(st, lib.gdr2_last_error().decode(errors="replace"))


def gdr2_abi_version() -> int:
    """GDR2_ABI_VERSION of the loaded libgdr2.so."""
    return load_library().gdr2_abi_version()


def gdr2_last_error() -> str:
    """Description of the calling thread's last non-OK status ('' if none)."""
    return load_library().gdr2_last_error().decode(errors="replace")


def gdr2_sync_status(stream=None) -> None:
    """Synchronise the stream and raise if a kernel gave up a bounded wait."""
    lib = load_library()
    _raise(lib, lib.gdr2_sync_status(_stream(stream)))


def gdr2_forward_workspace_bytes(B, T, H, dk, dv, dtype=torch.bfloat16) -> int:
    """Device scratch gdr2_forward needs (0 on the CUDA-core path: fp32, or d other than 128)."""
    lib = load_library()
    return int(lib.gdr2_forward_workspace_bytes(B, T, H, dk, dv, GDR2_BF16 if dtype == torch.bfloat16 else GDR2_F32))


@_one_device
def gdr2_forward(q, k, v, log_alpha, b, w, S0=None, *, final_state=True, save_states=False,
                 out=None, workspace=None, stream=None, out_gate=None, norm_weight=None, norm_eps=1e-6):
    """Chunkwise forward. Returns (o, S_T, saved_states); S_T / saved_states may be None.

    q, k, b: [B, T, H, dk]; v, w: [B, T, H, dv] (fp32 or bf16, one dtype);
    log_alpha: [B, T, H, dk] fp32; S0: [B, H, dk, dv] fp32 or None.
    b and/or w may instead be [B, T, H]: one gate value per token-head (scalar gates).
    out_gate ([B, T, H, dv], o's dtype) and norm_weight ([dv] fp32) apply the block's output
    epilogue o / rms(o) * norm_weight * silu(out_gate) in the kernel (bf16, d = 128 only).
    """
    lib = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    gates = _gates(b, w, (B, T, H))
    for name, t, shp in (("q", q, (B, T, H, dk)), ("k", k, (B, T, H, dk)),
                         ("b", b, (B, T, H) if gates & GATE_SCALAR_B else (B, T, H, dk)),
                         ("v", v, (B, T, H, dv)), ("w", w, (B, T, H) if gates & GATE_SCALAR_W else (B, T, H, dv))):
        _check(t, name, shp, dt)
    _check(log_alpha, "log_alpha", (B, T, H, dk), torch.float32)
    _check(S0, "S0", (B, H, dk, dv), torch.float32)
    dev = q.device
    o = out if out is not None else torch.empty((B, T, H, dv), dtype=dt, device=dev)
    _check(o, "o", (B, T, H, dv), dt)
    S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev) if final_state else None
    nc = (T + CHUNK - 1) // CHUNK
    saved = torch.empty((B, H, nc, dk, dv), dtype=torch.float32, device=dev) if save_states else None
    need = gdr2_forward_workspace_bytes(B, T, H, dk, dv, dt)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if _epilogue(out_gate, norm_weight, (B, T, H, dv), dv, dt, dev):
        st = lib.gdr2_forward_ex(B, T, H, dk, dv, _dt(q), gates, None, _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                                 _ptr(b), _ptr(w), _ptr(S0), _ptr(out_gate), _ptr(norm_weight),
                                 ctypes.c_float(norm_eps), _ptr(o), _ptr(S_T), _ptr(saved), _ptr(workspace),
                                 ctypes.c_size_t(ws_bytes), _stream(stream))
    else:
        st = lib.gdr2_forward_gated(B, T, H, dk, dv, _dt(q), gates, _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                                    _ptr(b), _ptr(w), _ptr(S0), _ptr(o), _ptr(S_T), _ptr(saved), _ptr(workspace),
                                    ctypes.c_size_t(ws_bytes), _stream(stream))
    _raise(lib, st)
    return o, S_T, saved


def gdr2_forward_varlen_workspace_bytes(N, T, H, dk, dv, dtype=torch.bfloat16) -> int:
    """Device scratch gdr2_forward_varlen needs for N sequences of T tokens in all."""
    lib = load_library()
    return int(lib.gdr2_forward_varlen_workspace_bytes(N, T, H, dk, dv,
                                                       GDR2_BF16 if dtype == torch.bfloat16 else GDR2_F32))


@_one_device
def gdr2_forward_varlen(q, k, v, log_alpha, b, w, cu_seqlens, S0=None, *, final_state=True, save_states=False,
                        out=None, workspace=None, stream=None, out_gate=None, norm_weight=None, norm_eps=1e-6):
    """Forward over packed sequences. Returns (o, S_T, saved_states).

    q, k, b: [T, H, dk] (or [1, T, H, dk]); v, w: [T, H, dv]; bf16; log_alpha [T, H, dk] fp32;
    cu_seqlens: int32 [N + 1] on the device; S0: [N, H, dk, dv] fp32 or None; b and/or w may
    be [T, H] (scalar gates). saved_states,
    when asked for, is [H * (ceil(T / 64) + N), dk, dv] (see include/gdr2.h for the order).
    out_gate ([T, H, dv] bf16) and norm_weight ([dv] fp32): the output epilogue, as in gdr2_forward.
    """
    lib = load_library()
    sq4 = lambda t: None if t is None else (t[0] if t.dim() == 4 else t)  # noqa: E731
    q, k, v, log_alpha = (sq4(t) for t in (q, k, v, log_alpha))
    T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    sqg = lambda t: t[0] if t.dim() == 4 or (t.dim() == 3 and tuple(t.shape) == (1, T, H)) else t  # noqa: E731
    b, w = sqg(b), sqg(w)
    gates = _gates(b, w, (T, H))
    for name, t, shp in (("q", q, (T, H, dk)), ("k", k, (T, H, dk)),
                         ("b", b, (T, H) if gates & GATE_SCALAR_B else (T, H, dk)),
                         ("v", v, (T, H, dv)), ("w", w, (T, H) if gates & GATE_SCALAR_W else (T, H, dv))):
        _check(t, name, shp, dt)
    _check(log_alpha, "log_alpha", (T, H, dk), torch.float32)
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or not cu_seqlens.is_contiguous() \
            or cu_seqlens.device != q.device:
        raise ValueError("cu_seqlens must be a contiguous 1-D int32 tensor on the inputs' device")
    N = cu_seqlens.numel() - 1
    _check(S0, "S0", (N, H, dk, dv), torch.float32)
    dev = q.device
    o = out if out is not None else torch.empty((T, H, dv), dtype=dt, device=dev)
    _check(sq4(o), "o", (T, H, dv), dt)
    S_T = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev) if final_state else None
    cap = H * ((T + CHUNK - 1) // CHUNK + N)
    saved = torch.empty((cap, dk, dv), dtype=torch.float32, device=dev) if save_states else None
    need = gdr2_forward_varlen_workspace_bytes(N, T, H, dk, dv, dt)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    out_gate = sq4(out_gate)
    if _epilogue(out_gate, norm_weight, (T, H, dv), dv, dt, dev):
        st = lib.gdr2_forward_ex(N, T, H, dk, dv, _dt(q), gates, _ptr(cu_seqlens), _ptr(q), _ptr(k), _ptr(v),
                                 _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(S0), _ptr(out_gate), _ptr(norm_weight),
                                 ctypes.c_float(norm_eps), _ptr(o), _ptr(S_T), _ptr(saved), _ptr(workspace),
                                 ctypes.c_size_t(ws_bytes), _stream(stream))
    else:
        st = lib.gdr2_forward_varlen(N, T, H, dk, dv, _dt(q), gates, _ptr(cu_seqlens), _ptr(q), _ptr(k), _ptr(v),
                                     _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(S0), _ptr(o), _ptr(S_T), _ptr(saved),
                                     _ptr(workspace), ctypes.c_size_t(ws_bytes), _stream(stream))
    _raise(lib, st)
    return o, S_T, saved


def _check_cu_seqlens(cu_seqlens, device):
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or not cu_seqlens.is_contiguous() \
            or cu_seqlens.device != device:
        raise ValueError("cu_seqlens must be a contiguous 1-D int32 tensor on the inputs' device")


@_one_device
def gdr2_short_conv_silu(x, weight, state=None, *, l2norm=False, eps=1e-6, cu_seqlens=None, final_state=False,
                         state_out=None, out=None, stream=None):
    """Block prologue of one branch: SiLU(causal depthwise convolution of x), then with
    l2norm the per-head L2 norm (query and key); without it, the value branch.

    x: [N, T, H, d] (dense) or [T, H, d] with cu_seqlens ([N + 1] int32); weight: [H * d, W]
    fp32 (a depthwise Conv1d weight [H * d, 1, W] too; the last tap is the current token);
    state: [N, W - 1, H, d] in x's dtype, the inputs before each sequence, or None (zeros).
    Returns (y, state_out): the state after the call when final_state or when a state_out
    tensor is given (state_out=state updates a decode step's state in place, T = 1), else None.
    """
    lib = load_library()
    if cu_seqlens is not None:
        T, H, d = x.shape
        _check_cu_seqlens(cu_seqlens, x.device)
        N = cu_seqlens.numel() - 1
    else:
        N, T, H, d = x.shape
    wgt = weight.reshape(weight.shape[0], weight.shape[-1]) if weight.dim() == 3 else weight
    W = int(wgt.shape[-1])
    dt = x.dtype
    _check(x, "x", tuple(x.shape), dt)
    _check(wgt, "weight", (H * d, W), torch.float32)
    _check(state, "state", (N, W - 1, H, d), dt)
    y = out if out is not None else torch.empty_like(x)
    _check(y, "out", tuple(x.shape), dt)
    if state_out is None and final_state:
        state_out = torch.empty((N, W - 1, H, d), dtype=dt, device=x.device)
    _check(state_out, "state_out", (N, W - 1, H, d), dt)
    ptr = lambda t: None if t is None or t.numel() == 0 else _ptr(t)  # noqa: E731
    st = lib.gdr2_short_conv_silu(N, T, H, d, _dt(x), W, int(bool(l2norm)), ctypes.c_float(eps), _ptr(cu_seqlens),
                                  ptr(x), ptr(wgt), ptr(state), ptr(state_out), ptr(y), _stream(stream))
    _raise(lib, st)
    return y, state_out


@_one_device
def gdr2_gate_activations(a=None, b=None, w=None, *, stream=None):
    """The decay and gate branches' activations, element by element, any of them None:
    log_alpha = -softplus(a) (fp32), sigmoid(b) and sigmoid(w) in the inputs' dtype."""
    lib = load_library()
    given = [t for t in (a, b, w) if t is not None]
    if not given:
        return None, None, None
    dt = given[0].dtype
    for name, t in (("a", a), ("b", b), ("w", w)):
        if t is not None:
            _check(t, name, tuple(t.shape), dt)
    la = None if a is None else torch.empty(tuple(a.shape), dtype=torch.float32, device=a.device)
    bo = None if b is None else torch.empty_like(b)
    wo = None if w is None else torch.empty_like(w)
    n = lambda t: 0 if t is None else t.numel()  # noqa: E731
    st = lib.gdr2_gate_activations(_dt(given[0]), n(a), _ptr(a), _ptr(la), n(b), _ptr(b), _ptr(bo), n(w), _ptr(w),
                                   _ptr(wo), _stream(stream))
    _raise(lib, st)
    return la, bo, wo


@_one_device
def gdr2_block_prologue(xq, xk, xv, conv_q, conv_k, conv_v, a, b, w, *, states=None, eps=1e-6, cu_seqlens=None,
                        final_state=False, stream=None):
    """The whole prologue: q, k = L2(SiLU(conv(x))) per head, v = SiLU(conv(x)), and the
    activations of a, b, w. states: (state_q, state_k, state_v) or None. Returns
    (q, k, v, log_alpha, b, w, new_states); new_states is a triple when final_state, else None."""
    sq, sk, sv = states if states is not None else (None, None, None)
    kw = dict(eps=eps, cu_seqlens=cu_seqlens, final_state=final_state, stream=stream)
    q, nq = gdr2_short_conv_silu(xq, conv_q, sq, l2norm=True, **kw)
    k, nk = gdr2_short_conv_silu(xk, conv_k, sk, l2norm=True, **kw)
    v, nv = gdr2_short_conv_silu(xv, conv_v, sv, l2norm=False, **kw)
    la, bo, wo = gdr2_gate_activations(a, b, w, stream=stream)
    return q, k, v, la, bo, wo, ((nq, nk, nv) if final_state else None)


@_one_device
def gdr2_segment_states(A, Bst, S0=None, *, final_state=True, stream=None):
    """States entering the segments of split sequences (see include/gdr2.h).

    A: [B, G, H, dk, dk] fp32 segment transitions; Bst: [B, G, H, dk, dv] fp32 segment
    offsets; S0: [B, H, dk, dv] fp32 or None. Returns (S_starts [B, G, H, dk, dv], S_T or None).
    """
    lib = load_library()
    B, G, H, dk, dv = Bst.shape
    _check(A, "A", (B, G, H, dk, dk), torch.float32)
    _check(Bst, "Bst", (B, G, H, dk, dv), torch.float32)
    _check(S0, "S0", (B, H, dk, dv), torch.float32)
    S_starts = torch.empty_like(Bst)
    S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=Bst.device) if final_state else None
    st = lib.gdr2_segment_states(B, G, H, dk, dv, _ptr(A), _ptr(Bst), _ptr(S0), _ptr(S_starts), _ptr(S_T),
                                 _stream(stream))
    _raise(lib, st)
    return S_starts, S_T


@_one_device
def gdr2_decode_step(q, k, v, log_alpha, b, w, S, *, out=None, stream=None):
    """One decode token; S [N, H, dk, dv] fp32 is updated in place. Returns o [N, H, dv].

    b and/or w may be [N, H]: one gate value per token-head (scalar gates).
    """
    lib = load_library()
    N, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    gates = _gates(b, w, (N, H))
    for name, t, shp in (("q", q, (N, H, dk)), ("k", k, (N, H, dk)),
                         ("b", b, (N, H) if gates & GATE_SCALAR_B else (N, H, dk)),
                         ("v", v, (N, H, dv)), ("w", w, (N, H) if gates & GATE_SCALAR_W else (N, H, dv))):
        _check(t, name, shp, dt)
    _check(log_alpha, "log_alpha", (N, H, dk), torch.float32)
    _check(S, "S", (N, H, dk, dv), torch.float32)
    o = out if out is not None else torch.empty((N, H, dv), dtype=dt, device=q.device)
    _check(o, "o", (N, H, dv), dt)
    st = lib.gdr2_decode_step_gated(N, H, dk, dv, _dt(q), gates, _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                                    _ptr(b), _ptr(w), _ptr(S), _ptr(o), _stream(stream))
    _raise(lib, st)
    return o


def gdr2_backward_workspace_bytes(B, T, H, dk, dv, dtype=torch.bfloat16) -> int:
    """Device scratch gdr2_backward needs for this problem."""
    lib = load_library()
    return int(lib.gdr2_backward_workspace_bytes(B, T, H, dk, dv, GDR2_BF16 if dtype == torch.bfloat16 else GDR2_F32))


@_one_device
def gdr2_backward(q, k, v, log_alpha, b, w, dO, S0=None, dS_T=None, saved_states=None, *,
                  want_dS0=True, workspace=None, stream=None):
    """Gradients of <o, dO> + <S_T, dS_T>. Returns dict dq, dk, dv, dlog_alpha, db, dw, dS0.

    b or w shaped [B, T, H] (one value per token-head) are scalar gates; their gradients
    have the same shape (the tensor-core path: bf16 with dk = dv = 128).
    """
    lib = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    gates = _gates(b, w, (B, T, H))
    for name, t, shp in (("q", q, (B, T, H, dk)), ("k", k, (B, T, H, dk)),
                         ("b", b, (B, T, H) if gates & GATE_SCALAR_B else (B, T, H, dk)),
                         ("v", v, (B, T, H, dv)), ("w", w, (B, T, H) if gates & GATE_SCALAR_W else (B, T, H, dv)),
                         ("dO", dO, (B, T, H, dv))):
        _check(t, name, shp, dt)
    _check(log_alpha, "log_alpha", (B, T, H, dk), torch.float32)
    _check(S0, "S0", (B, H, dk, dv), torch.float32)
    _check(dS_T, "dS_T", (B, H, dk, dv), torch.float32)
    nc = (T + CHUNK - 1) // CHUNK
    _check(saved_states, "saved_states", (B, H, nc, dk, dv), torch.float32)
    dev = q.device
    g = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
         "dlog_alpha": torch.empty_like(log_alpha), "db": torch.empty_like(b), "dw": torch.empty_like(w),
         "dS0": torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev) if want_dS0 else None}
    need = gdr2_backward_workspace_bytes(B, T, H, dk, dv, dt)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    st = lib.gdr2_backward_gated(B, T, H, dk, dv, _dt(q), gates, _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                                 _ptr(b), _ptr(w), _ptr(S0), _ptr(dO), _ptr(dS_T), _ptr(saved_states),
                                 _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dlog_alpha"]), _ptr(g["db"]),
                                 _ptr(g["dw"]), _ptr(g["dS0"]), _ptr(workspace), ctypes.c_size_t(workspace.numel()),
                                 _stream(stream))
    _raise(lib, st)
    return g


@_one_device
def gdr2_backward_noalloc(q, k, v, log_alpha, b, w, dO, S0=None, dS_T=None, saved_states=None, *,
                          want_dS0=True, stream=None):
    """gdr2_backward through the entry point that allocates nothing on the device.

    The library uses its own fixed scratch array (NOALLOC_SCRATCH_BYTES per
    device) instead of a workspace; the gradient tensors returned here are
    ordinary torch allocations made by this binding, not by the library.
    """
    lib = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = q.dtype
    for name, t, shp in (("q", q, (B, T, H, dk)), ("k", k, (B, T, H, dk)), ("b", b, (B, T, H, dk)),
                         ("v", v, (B, T, H, dv)), ("w", w, (B, T, H, dv)), ("dO", dO, (B, T, H, dv))):
        _check(t, name, shp, dt)
    _check(log_alpha, "log_alpha", (B, T, H, dk), torch.float32)
    _check(S0, "S0", (B, H, dk, dv), torch.float32)
    _check(dS_T, "dS_T", (B, H, dk, dv), torch.float32)
    nc = (T + CHUNK - 1) // CHUNK
    _check(saved_states, "saved_states", (B, H, nc, dk, dv), torch.float32)
    dev = q.device
    g = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
         "dlog_alpha": torch.empty_like(log_alpha), "db": torch.empty_like(b), "dw": torch.empty_like(w),
         "dS0": torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev) if want_dS0 else None}
    st = lib.gdr2_backward_noalloc(B, T, H, dk, dv, _dt(q), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                                   _ptr(b), _ptr(w), _ptr(S0), _ptr(dO), _ptr(dS_T), _ptr(saved_states),
                                   _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dlog_alpha"]),
                                   _ptr(g["db"]), _ptr(g["dw"]), _ptr(g["dS0"]), _stream(stream))
    _raise(lib, st)
    return g
