"""Oracle for the gated delta rule -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package. The CUDA product path never
imports it and shares no code with it.

Two independent fp64 CPU implementations live here:

* :func:`recurrence_fwd` / :func:`recurrence_decode_step` -- the plain
  token-by-token recurrence (the definition), in C (``gdr_oracle.c``), threaded
  over (sequence, head).  Sources: "Gated DeltaNet: Householder Transitions and
  the Arithmetic of Forgetting", section "The gated delta rule"; "Linear
  Attention, Visualized", sections "DeltaNet / Recurrent form", "Gated DeltaNet
  (GDN)" and "Kimi Delta Attention (KDA)".
* :func:`product_fwd` -- Gated DeltaProduct, token by token with n_h
  Householder substeps per token ("Linear Attention, Visualized", section
  "Gated Delta Product (GDP)"), written from that definition.
* :func:`gdn2_fwd` -- Gated DeltaNet-2 (decoupled erase and write gates),
  token by token ("Gated DeltaNet-2, and the gate that was doing two jobs",
  section "What decoupling actually means here"), and
  :func:`oracle.chunked.gdn2_chunked_fwd`, its chunkwise form from the same
  section, used only to pin it.
* :func:`frame_fwd` -- the implicit frame-level update ("video-delta-rule",
  section "A Different Route"): per frame of n tokens, Cholesky of I + G_t and
  a solve of S_t (I + G_t) = S_{t-1} D_t + C_t.
* :func:`oracle.chunked.chunked_fwd` -- the chunkwise WY/UT algorithm written
  from "Linear Attention, Visualized", sections "Gated DeltaNet (GDN) /
  Complete per-chunk algorithm" and "Kimi Delta Attention (KDA) / Complete
  per-chunk algorithm".  It is used only to pin the recurrence (the pages state
  that every chunk size gives the exact result).

Every function here is pinned by ``tests/test_oracle_pins.py`` against closed
forms, invariants and exact-rational brute force that the pages fix.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (strict IEEE fp64: no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared",
               "-o", _LIB, _SRC, "-lm", "-lpthread"]
        subprocess.check_call(cmd)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int)
            lib.oracle_gdr_fwd.restype = ctypes.c_int
            lib.oracle_gdr_fwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ip, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int]
            lib.oracle_gdp_fwd.restype = ctypes.c_int
            lib.oracle_gdp_fwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ip, ctypes.c_int, ctypes.c_int]
            lib.oracle_gdn2_fwd.restype = ctypes.c_int
            lib.oracle_gdn2_fwd.argtypes = [dp] * 9 + [ctypes.c_int] * 5 + [ip, ctypes.c_int,
                                                                             ctypes.c_int]
            lib.oracle_frame_fwd.restype = ctypes.c_int
            lib.oracle_frame_fwd.argtypes = [dp] * 8 + [ctypes.c_int] * 7
            lib.oracle_gdr_decode_step.restype = ctypes.c_int
            lib.oracle_gdr_decode_step.argtypes = [dp, dp, dp, dp, dp, dp, dp,
                                                   ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_int, ctypes.c_int]
            _lib = lib
    return _lib


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def recurrence_fwd(q, k, v, g, beta, S0=None, cu_seqlens=None, threads=None):
    """Token-by-token fp64 recurrence over whole sequences.

    Shapes: q, k ``[B, T, H, d_k]``; v ``[B, T, H, d_v]``; g ``[B, T, H]``
    (scalar gate) or ``[B, T, H, d_k]`` (per-key-channel gate), the log of the
    decay; beta ``[B, T, H]``; S0 ``[N, H, d_v, d_k]`` or None (zero state).
    With ``cu_seqlens`` (length N+1 token offsets) B must be 1 and the state is
    reset at every sequence boundary.  Returns ``(O [B,T,H,d_v], S_final
    [N,H,d_v,d_k])`` in float64.
    """
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    per_channel = 1 if g.ndim == 4 else 0
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        n_seq = len(cu) - 1
        cu_p = cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int))
    else:
        cu = None
        n_seq = B
        cu_p = None
    S0a = None if S0 is None else _f64(S0)
    out = np.zeros((B, T, H, dv), dtype=np.float64)
    S_final = np.zeros((n_seq, H, dv, dk), dtype=np.float64)
    rc = _load().oracle_gdr_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0a),
                                _ptr(out), _ptr(S_final), B, T, H, dk, dv, cu_p, n_seq,
                                per_channel, int(threads or default_threads()))
    if rc != 0:
        raise ValueError("oracle_gdr_fwd rejected its arguments")
    return out, S_final


def recurrence_decode_step(q, k, v, g, beta, S):
    """One decode step for N sequences; returns ``(out [N,H,d_v], S_new)``.

    q, k ``[N, H, d_k]``; v ``[N, H, d_v]``; g ``[N, H]`` or ``[N, H, d_k]``;
    beta ``[N, H]``; S ``[N, H, d_v, d_k]`` (not modified; a copy is updated).
    """
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    S_new = _f64(S).copy()
    N, H, dk = q.shape
    dv = v.shape[-1]
    out = np.zeros((N, H, dv), dtype=np.float64)
    rc = _load().oracle_gdr_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                        _ptr(S_new), _ptr(out), N, H, dk, dv,
                                        1 if g.ndim == 3 else 0)
    if rc != 0:
        raise ValueError("oracle_gdr_decode_step rejected its arguments")
    return out, S_new


def product_fwd(q, k, v, g, beta, S0=None, cu_seqlens=None):
    """Gated DeltaProduct, fp64.  q ``[B,T,H,d_k]``; k ``[B,T,n_h,H,d_k]``;
    v ``[B,T,n_h,H,d_v]``; g ``[B,T,H]`` or ``[B,T,H,d_k]``; beta
    ``[B,T,n_h,H]``.  Returns ``(O [B,T,H,d_v], S_final [N,H,d_v,d_k])``."""
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    B, T, H, dk = q.shape
    nh = k.shape[2]
    dv = v.shape[-1]
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        n_seq = len(cu) - 1
        cu_p = cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int))
    else:
        cu, n_seq, cu_p = None, B, None
    S0a = None if S0 is None else _f64(S0)
    out = np.zeros((B, T, H, dv))
    S_final = np.zeros((n_seq, H, dv, dk))
    rc = _load().oracle_gdp_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0a),
                                _ptr(out), _ptr(S_final), B, T, H, nh, dk, dv, cu_p, n_seq,
                                1 if g.ndim == 4 else 0)
    if rc != 0:
        raise ValueError("oracle_gdp_fwd rejected its arguments")
    return out, S_final


def gdn2_fwd(q, k, v, g, b, w, S0=None, cu_seqlens=None):
    """Gated DeltaNet-2, fp64.  q, k ``[B,T,H,d_k]``; v ``[B,T,H,d_v]``; g
    ``[B,T,H]`` or ``[B,T,H,d_k]``; erase gate b ``[B,T,H,d_k]``; write gate w
    ``[B,T,H,d_v]``.  Returns ``(O [B,T,H,d_v], S_final [N,H,d_v,d_k])``."""
    q, k, v, g, b, w = (_f64(x) for x in (q, k, v, g, b, w))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        n_seq = len(cu) - 1
        cu_p = cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int))
    else:
        cu, n_seq, cu_p = None, B, None
    S0a = None if S0 is None else _f64(S0)
    out = np.zeros((B, T, H, dv))
    S_final = np.zeros((n_seq, H, dv, dk))
    rc = _load().oracle_gdn2_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), _ptr(S0a),
                                 _ptr(out), _ptr(S_final), B, T, H, dk, dv, cu_p, n_seq,
                                 1 if g.ndim == 4 else 0)
    if rc != 0:
        raise ValueError("oracle_gdn2_fwd rejected its arguments")
    return out, S_final


def frame_fwd(q, k, v, g, gamma, n, S0=None):
    """Implicit frame-level update, fp64.  q, k ``[B,T,H,d_k]``; v ``[B,T,H,d_v]``;
    gamma ``[B,T,H]`` (writing strength); g ``[B,F,H]`` or ``[B,F,H,d_k]`` with
    F = ceil(T / n) (log-decay per frame).  Returns ``(O [B,T,H,d_v], S_final
    [B,H,d_v,d_k])``."""
    q, k, v, g, gamma = (_f64(x) for x in (q, k, v, g, gamma))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    S0a = None if S0 is None else _f64(S0)
    out = np.zeros((B, T, H, dv))
    S_final = np.zeros((B, H, dv, dk))
    rc = _load().oracle_frame_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(gamma), _ptr(S0a),
                                  _ptr(out), _ptr(S_final), B, T, H, dk, dv, int(n),
                                  1 if g.ndim == 4 else 0)
    if rc != 0:
        raise ValueError("oracle_frame_fwd rejected its arguments (%d)" % rc)
    return out, S_final
