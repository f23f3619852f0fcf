"""float64 CPU oracle for chunkwise Gated Linear Attention -- ctypes front end.

TEST INFRASTRUCTURE ONLY.  The product path (``chunkwise_linear_rnn_fwd_b200``)
never imports this module; only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` do.

The arithmetic lives in ``gla_oracle.c`` (the literal token recurrence of
"Gated Linear Attention Transformers with Hardware-Efficient Training",
section 4.1, its general-gate form of appendix C, and back-propagation through
them).  This module compiles that file
with the host C compiler on first use and marshals numpy float64 arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

GATE_VECTOR = 0
GATE_SCALAR = 1
GATE_NONE = 2
_GATE_NAMES = {"vector": GATE_VECTOR, "scalar": GATE_SCALAR, "none": GATE_NONE}

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gla_oracle.c")
_LIB = os.path.join(_HERE, "libgla_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False, mutant: int = 0) -> str:
    """Compile gla_oracle.c into libgla_oracle.so (gcc, -O2, OpenMP).
    mutant > 0 builds a planted-mistake variant (pin tests only)."""
    out = _LIB if mutant == 0 else os.path.join(_HERE, f"libgla_oracle_mutant{mutant}.so")
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(_SRC):
        tmp = out + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
               f"-DGLA_ORACLE_MUTANT={int(mutant)}", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return out


def _open(path):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.gla_oracle_fwd.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_long, ctypes.c_int,
                                   ctypes.c_int, ctypes.c_int, dp, dp, dp, dp, dp, dp, dp]
    lib.gla_oracle_fwd.restype = None
    lib.gla_oracle_bwd.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_long, ctypes.c_int,
                                   ctypes.c_int, ctypes.c_int, dp, dp, dp, dp, dp, dp, dp,
                                   dp, dp, dp, dp, dp]
    lib.gla_oracle_bwd.restype = None
    lib.gla_oracle_fwd_general.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_long, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, dp, dp, dp, dp, dp, dp, dp, dp]
    lib.gla_oracle_fwd_general.restype = None
    lib.gla_oracle_bwd_general.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_long, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, dp, dp, dp, dp, dp, dp, dp, dp,
                                           dp, dp, dp, dp, dp, dp]
    lib.gla_oracle_bwd_general.restype = None
    lib.gla_oracle_max_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = _open(build())
            _lib = lib
    return _lib


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    if a is None:
        return None
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _gate_mode(gate):
    return _GATE_NAMES[gate] if isinstance(gate, str) else int(gate)


def threads() -> int:
    """OpenMP threads the oracle runs its (batch, head) loop on."""
    return int(_load().gla_oracle_max_threads())


def fwd(q, k, v, log_alpha, h0=None, gate="vector", _lib_override=None):
    """Recurrent-form forward.  Shapes: q,k [B,H,T,K]; v [B,H,T,V];
    log_alpha [B,H,T,K] (vector) / [B,H,T] (scalar) / None (none).
    Returns (o [B,H,T,V], h_final [B,H,K,V]) as float64."""
    mode = _gate_mode(gate)
    q, k, v, la, h0 = _f64(q), _f64(k), _f64(v), _f64(log_alpha), _f64(h0)
    B, H, T, K = q.shape
    V = v.shape[-1]
    o = np.empty((B, H, T, V), np.float64)
    hT = np.empty((B, H, K, V), np.float64)
    if mode == GATE_NONE:
        la = None
    (_lib_override or _load()).gla_oracle_fwd(B, H, T, K, V, mode, _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(h0),
                           _ptr(o), _ptr(hT))
    return o, hT


def bwd(q, k, v, log_alpha, do, h0=None, dh_final=None, gate="vector", _lib_override=None):
    """Back-propagation through the recurrence.  Returns
    (dq, dk, dv, dlog_alpha or None, dh0) as float64."""
    mode = _gate_mode(gate)
    q, k, v, la, do = _f64(q), _f64(k), _f64(v), _f64(log_alpha), _f64(do)
    h0, dhT = _f64(h0), _f64(dh_final)
    B, H, T, K = q.shape
    V = v.shape[-1]
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    if mode == GATE_VECTOR:
        dla = np.empty((B, H, T, K), np.float64)
    elif mode == GATE_SCALAR:
        dla = np.empty((B, H, T), np.float64)
    else:
        dla, la = None, None
    dh0 = np.empty((B, H, K, V), np.float64)
    (_lib_override or _load()).gla_oracle_bwd(B, H, T, K, V, mode, _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(h0),
                           _ptr(do), _ptr(dhT), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dla), _ptr(dh0))
    return dq, dk, dv, dla, dh0


def fwd_general(q, k, v, log_alpha, log_beta, h0=None, gate="vector", _lib_override=None):
    """Recurrent form with the general gate G_t = alpha_t^T beta_t (appendix C):
    S_t = diag(alpha_t) S_{t-1} diag(beta_t) + k_t^T v_t, o_t = q_t S_t.
    log_beta [B,H,T,V] (None: beta == 1).  Returns (o, h_final) as float64."""
    mode = _gate_mode(gate)
    q, k, v, la, lb, h0 = _f64(q), _f64(k), _f64(v), _f64(log_alpha), _f64(log_beta), _f64(h0)
    B, H, T, K = q.shape
    V = v.shape[-1]
    o = np.empty((B, H, T, V), np.float64)
    hT = np.empty((B, H, K, V), np.float64)
    if mode == GATE_NONE:
        la = None
    (_lib_override or _load()).gla_oracle_fwd_general(B, H, T, K, V, mode, _ptr(q), _ptr(k), _ptr(v), _ptr(la),
                                                      _ptr(lb), _ptr(h0), _ptr(o), _ptr(hT))
    return o, hT


def bwd_general(q, k, v, log_alpha, log_beta, do, h0=None, dh_final=None, gate="vector", _lib_override=None):
    """Back-propagation through the general-gate recurrence.  Returns
    (dq, dk, dv, dlog_alpha or None, dlog_beta or None, dh0) as float64."""
    mode = _gate_mode(gate)
    q, k, v, la, lb, do = _f64(q), _f64(k), _f64(v), _f64(log_alpha), _f64(log_beta), _f64(do)
    h0, dhT = _f64(h0), _f64(dh_final)
    B, H, T, K = q.shape
    V = v.shape[-1]
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    if mode == GATE_VECTOR:
        dla = np.empty((B, H, T, K), np.float64)
    elif mode == GATE_SCALAR:
        dla = np.empty((B, H, T), np.float64)
    else:
        dla, la = None, None
    dlb = None if lb is None else np.empty((B, H, T, V), np.float64)
    dh0 = np.empty((B, H, K, V), np.float64)
    (_lib_override or _load()).gla_oracle_bwd_general(B, H, T, K, V, mode, _ptr(q), _ptr(k), _ptr(v), _ptr(la),
                                                      _ptr(lb), _ptr(h0), _ptr(do), _ptr(dhT), _ptr(dq), _ptr(dk),
                                                      _ptr(dv), _ptr(dla), _ptr(dlb), _ptr(dh0))
    return dq, dk, dv, dla, dlb, dh0


def decode_step(q, k, v, log_alpha, state, gate="vector"):
    """One recurrent decode step per (batch, head): the recurrence of section 4.1 at a
    single token, S <- diag(alpha) S + k^T v, o = q S (the state after the update).
    Shapes: q, k [B,H,K]; v [B,H,V]; log_alpha [B,H,K] (vector) / [B,H] (scalar) /
    None (none); state [B,H,K,V] (None = zero).  Returns (o [B,H,V], new state
    [B,H,K,V]) as float64; `state` itself is not modified."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    la = None if log_alpha is None else _f64(log_alpha)[:, :, None]
    o, hT = fwd(q[:, :, None], k[:, :, None], v[:, :, None], la, h0=state, gate=gate)
    return o[:, :, 0], hT


class Mutant:
    """A planted-mistake build of the oracle (pin tests only)."""

    def __init__(self, n: int):
        self._lib = _open(build(mutant=n))

    def fwd(self, *a, **kw):
        return fwd(*a, _lib_override=self._lib, **kw)

    def bwd(self, *a, **kw):
        return bwd(*a, _lib_override=self._lib, **kw)

    def fwd_general(self, *a, **kw):
        return fwd_general(*a, _lib_override=self._lib, **kw)

    def bwd_general(self, *a, **kw):
        return bwd_general(*a, _lib_override=self._lib, **kw)
