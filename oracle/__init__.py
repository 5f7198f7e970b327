"""fp64 CPU oracle for the Gated Delta Rule-2 token mixer (test infrastructure).

This package is the checker, not the product. Only ``tests/``, the smoke check
in ``__graft_entry__.py`` and the CPU-baseline leg of ``bench.py`` may import
it. It shares no code with the CUDA library: the arithmetic lives in
``gdr2_oracle.c`` (plain C, fp64, token by token, OpenMP over (batch, head)),
and this module only marshals numpy arrays through ctypes.

Source of the recurrence: "Gated DeltaNet-2: Decoupling Erase and Write in
Linear Attention" (graygoo.forestry.md note), sec. 2 fast-weight objective and
sec. 3 forward-pass and gate-aware-backward paragraphs; the C file's header
states the update and the reading of the erase outer product.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr2_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libgdr2_oracle.so")
_lock = threading.Lock()
_lib = None

_D = ctypes.POINTER(ctypes.c_double)


def compile_library(src: str, out: str) -> str:
    """Compile one oracle C source into a shared library (gcc, -O2, OpenMP)."""
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC", "-Wall", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile ``gdr2_oracle.c`` into ``libgdr2_oracle.so`` when missing or stale."""
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC):
        return _LIB_PATH
    return compile_library(_SRC, _LIB_PATH)


class OracleLib:
    """ctypes front end of one compiled oracle library."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        I = ctypes.c_int
        lib.gdr2_oracle_forward.argtypes = [I, I, I, I, I] + [_D] * 9 + [I]
        lib.gdr2_oracle_decode_step.argtypes = [I, I, I, I] + [_D] * 8 + [I]
        lib.gdr2_oracle_backward.argtypes = [I, I, I, I, I] + [_D] * 16 + [I]
        for f in (lib.gdr2_oracle_forward, lib.gdr2_oracle_decode_step, lib.gdr2_oracle_backward):
            f.restype = I
        self.lib = lib
        self.path = path

    def forward(self, *a, **kw):
        return _forward(self.lib, *a, **kw)

    def decode_step(self, *a, **kw):
        return _decode_step(self.lib, *a, **kw)

    def backward(self, *a, **kw):
        return _backward(self.lib, *a, **kw)


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = OracleLib(build())
    return _lib


def default_oracle() -> OracleLib:
    return _load()


def _in(x):
    """Read-only fp64 C-contiguous view (None passes through as NULL)."""
    if x is None:
        return None, None
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    return a, a.ctypes.data_as(_D)


def _out(shape):
    a = np.zeros(shape, dtype=np.float64)
    return a, a.ctypes.data_as(_D)


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _forward(lib, q, k, v, log_alpha, b, w, S0=None, nthreads: int | None = None, want_o: bool = True):
    """Token-by-token GDR-2 forward.

    q, k, log_alpha, b: [B, T, H, dk]; v, w: [B, T, H, dv]; S0: [B, H, dk, dv] or None.
    Returns (o [B, T, H, dv], S_T [B, H, dk, dv]) as float64 arrays (o is None
    when ``want_o`` is False).
    """
    q_, pq = _in(q)
    B, T, H, dk = q_.shape
    dv = np.asarray(v).shape[-1]
    k_, pk = _in(k)
    v_, pv = _in(v)
    la_, pla = _in(log_alpha)
    b_, pb = _in(b)
    w_, pw = _in(w)
    s0_, ps0 = _in(S0)
    o, po = _out((B, T, H, dv)) if want_o else (None, None)
    sT, psT = _out((B, H, dk, dv))
    rc = lib.gdr2_oracle_forward(B, T, H, dk, dv, pq, pk, pv, pla, pb, pw, ps0, po, psT,
                               nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"gdr2_oracle_forward failed with code {rc}")
    return o, sT


def _decode_step(lib, q, k, v, log_alpha, b, w, S, nthreads: int | None = None):
    """One recurrent step on N*H resident states.

    q, k, log_alpha, b: [N, H, dk]; v, w: [N, H, dv]; S: [N, H, dk, dv].
    Returns (o [N, H, dv], S_new [N, H, dk, dv]); the input S is not modified.
    """
    q_, pq = _in(q)
    N, H, dk = q_.shape
    dv = np.asarray(v).shape[-1]
    k_, pk = _in(k)
    v_, pv = _in(v)
    la_, pla = _in(log_alpha)
    b_, pb = _in(b)
    w_, pw = _in(w)
    S_new = np.array(S, dtype=np.float64, copy=True, order="C")
    o, po = _out((N, H, dv))
    rc = lib.gdr2_oracle_decode_step(N, H, dk, dv, pq, pk, pv, pla, pb, pw,
                                         S_new.ctypes.data_as(_D), po, nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"gdr2_oracle_decode_step failed with code {rc}")
    return o, S_new


def _backward(lib, q, k, v, log_alpha, b, w, dO, S0=None, dS_T=None, nthreads: int | None = None):
    """Reverse-mode gradients of the token recurrence.

    Returns a dict with dq, dk, dv, dlog_alpha, db, dw (input layouts) and dS0.
    """
    q_, pq = _in(q)
    B, T, H, dk = q_.shape
    dv = np.asarray(v).shape[-1]
    k_, pk = _in(k)
    v_, pv = _in(v)
    la_, pla = _in(log_alpha)
    b_, pb = _in(b)
    w_, pw = _in(w)
    s0_, ps0 = _in(S0)
    dO_, pdO = _in(dO)
    dsT_, pdsT = _in(dS_T)
    dq, pdq = _out((B, T, H, dk))
    dkk, pdk = _out((B, T, H, dk))
    dvv, pdv = _out((B, T, H, dv))
    dla, pdla = _out((B, T, H, dk))
    db, pdb = _out((B, T, H, dk))
    dw, pdw = _out((B, T, H, dv))
    dS0, pdS0 = _out((B, H, dk, dv))
    rc = lib.gdr2_oracle_backward(B, T, H, dk, dv, pq, pk, pv, pla, pb, pw, ps0, pdO, pdsT,
                                      pdq, pdk, pdv, pdla, pdb, pdw, pdS0, nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"gdr2_oracle_backward failed with code {rc}")
    return {"dq": dq, "dk": dkk, "dv": dvv, "dlog_alpha": dla, "db": db, "dw": dw, "dS0": dS0}


def forward(*a, **kw):
    """Token-by-token forward with the default library; see ``_forward``."""
    return _load().forward(*a, **kw)


def decode_step(*a, **kw):
    """One decode step with the default library; see ``_decode_step``."""
    return _load().decode_step(*a, **kw)


def backward(*a, **kw):
    """Reverse-mode gradients with the default library; see ``_backward``."""
    return _load().backward(*a, **kw)
