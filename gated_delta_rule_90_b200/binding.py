"""ctypes binding of libgdr (include/gdr.h) for torch tensors.

Argument marshalling only: shapes are read off the tensors, outputs and the
workspace are allocated with torch, and every step of the computation runs
in libgdr's CUDA kernels.  There is no fallback: if the library is missing
the call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdr.so")
# The checked build (kernels guard their accesses; see gdr.h, gdr_checked_build).
CHECKED_LIB_PATH = os.path.join(_HERE, "libgdr_check.so")
# GDR_LIBRARY=<path> loads another build of the same library instead, e.g.
# CHECKED_LIB_PATH.
LIB_ENV = "GDR_LIBRARY"

GDR_OK, GDR_ERR_INVALID, GDR_ERR_UNSUPPORTED, GDR_ERR_CUDA, GDR_ERR_TIMEOUT, GDR_ERR_BOUNDS = \
    range(6)
GDR_F32, GDR_BF16 = 0, 1
GDR_GATE_SCALAR, GDR_GATE_PER_KEY_CHANNEL = 0, 1
PATHS = {"auto": 0, "simt": 1, "tc": 2}
KERNELS = {"decode": 0, "fwd_simt": 1, "tc_plan": 2, "tc_wy": 3, "tc_state": 4, "gdp_remap": 5,
           "gdn2_simt": 6, "gdn2_decode": 7, "frame_gram": 8, "frame_solve": 9, "frame_chain": 10,
           "frame_out": 11}

_lib = None


class GdrError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)}")


def library_path() -> str:
    """The library lib() loads: $GDR_LIBRARY if set, else libgdr.so."""
    return os.environ.get(LIB_ENV) or LIB_PATH


def lib() -> ctypes.CDLL:
    """Load libgdr.so (built in-tree by __graft_entry__.build())."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(f"{os.path.basename(path)} is not built ({path}); "
                               "run __graft_entry__.build()")
        L = ctypes.CDLL(path)
        vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.gdr_status_string.restype = ctypes.c_char_p
        L.gdr_status_string.argtypes = [i]
        L.gdr_fwd_workspace_size.restype = sz
        L.gdr_fwd_workspace_size.argtypes = [i, i, i, i, i, i, i, i, i, i, i]
        L.gdr_fwd.restype = i
        L.gdr_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, i, i, i, i,
                              vp, sz, vp]
        L.gdr_decode_step.restype = i
        L.gdr_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp]
        L.gdr_device_status.restype = i
        L.gdr_device_status.argtypes = [vp]
        L.gdr_selftest_wait_timeout.restype = i
        L.gdr_selftest_wait_timeout.argtypes = [ctypes.c_uint, vp]
        L.gdr_checked_build.restype = i
        L.gdr_checked_build.argtypes = []
        L.gdr_selftest_bounds.restype = i
        L.gdr_selftest_bounds.argtypes = [vp]
        L.gdr_fwd_product_workspace_size.restype = sz
        L.gdr_fwd_product_workspace_size.argtypes = [i] * 12
        L.gdr_fwd_product.restype = i
        L.gdr_fwd_product.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp, i,
                                      i, i, i, vp, sz, vp]
        L.gdr_fwd_gdn2.restype = i
        L.gdr_fwd_gdn2.argtypes = [vp] * 9 + [i] * 6 + [vp, i, i, i, i, vp, sz, vp]
        L.gdr_fwd_gdn2_workspace_size.restype = sz
        L.gdr_fwd_gdn2_workspace_size.argtypes = [i] * 11
        L.gdr_decode_step_gdn2.restype = i
        L.gdr_decode_step_gdn2.argtypes = [vp] * 8 + [i] * 6 + [vp]
        L.gdr_fwd_frame_workspace_size.restype = sz
        L.gdr_fwd_frame_workspace_size.argtypes = [i] * 6
        L.gdr_fwd_frame.restype = i
        L.gdr_fwd_frame.argtypes = [vp] * 8 + [i] * 8 + [vp, sz, vp]
        L.gdr_profile_enable.restype = None
        L.gdr_profile_enable.argtypes = [i]
        L.gdr_profile_read.restype = i
        L.gdr_profile_read.argtypes = [i, ctypes.POINTER(ctypes.c_longlong),
                                       ctypes.POINTER(ctypes.c_double)]
        L.gdr_set_gram_spread_limit.restype = ctypes.c_float
        L.gdr_set_gram_spread_limit.argtypes = [ctypes.c_float]
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().gdr_status_string(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device=None) -> ctypes.c_void_p:
    """The cudaStream_t handle of ``stream`` (None: the current stream of
    ``device``).  A torch stream must belong to ``device``: the library
    launches on the current device, which the calls below set to it."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    sdev = getattr(stream, "device", None)
    if device is not None and sdev is not None and torch.device(sdev) != torch.device(device):
        raise ValueError(f"stream belongs to {sdev}; the tensors are on {device}")
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _call_on(device, fn):
    """Run ``fn`` with ``device`` as the current CUDA device.  libgdr launches
    on the current device (its tensor maps, error word and scratch lookup are
    per device), so every call is made with the tensors' device current."""
    with torch.cuda.device(device):
        return fn()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDR_BF16
    if t.dtype == torch.float32:
        return GDR_F32
    raise TypeError(f"q/k/v must be float32 or bfloat16, got {t.dtype}")


def _need_contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _check(device, *specs):
    """The memory the kernels will read or write, checked before the call:
    each ``(name, tensor, dtype, numel)`` (tensor None = absent) must live on
    ``device``, have ``dtype`` (None: not checked) and hold at least ``numel``
    elements.  A tensor on another device, of a narrower type or too small
    would otherwise be addressed out of bounds by the kernels."""
    for name, t, dtype, numel in specs:
        if t is None:
            continue
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a torch.Tensor")
        if t.device != device:
            raise ValueError(f"{name} is on {t.device}; expected {device}")
        if dtype is not None and t.dtype != dtype:
            raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
        if t.numel() < numel:
            raise ValueError(f"{name} holds {t.numel()} elements; needs {numel}")


def _on_cuda(q):
    if not isinstance(q, torch.Tensor) or q.device.type != "cuda":
        raise ValueError("tensors must be CUDA tensors")
    return q.device


def fwd_workspace_size(B, T, H, d_k, d_v, chunk, n_seq, varlen, dtype, gate, path="auto") -> int:
    return int(lib().gdr_fwd_workspace_size(B, T, H, d_k, d_v, chunk, n_seq, int(bool(varlen)),
                                            dtype, gate, PATHS[path]))


def fwd_product_workspace_size(B, T, H, n_h, d_k, d_v, chunk, n_seq, varlen, dtype, gate,
                               path="auto") -> int:
    return int(lib().gdr_fwd_product_workspace_size(B, T, H, n_h, d_k, d_v, chunk, n_seq,
                                                    int(bool(varlen)), dtype, gate, PATHS[path]))


def gdr_fwd(q, k, v, g, beta, S0=None, *, chunk: int = 64, cu_seqlens=None, out=None,
            S_final=None, want_final: bool = True, path: str = "auto", workspace=None,
            stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Prefill: returns ``(out [B,T,H,d_v], S_final [N,H,d_v,d_k] or None)``."""
    B, T, H, d_k = q.shape
    d_v = v.shape[-1]
    dtype = _dtype_code(q)
    gate = GDR_GATE_PER_KEY_CHANNEL if g.dim() == 4 else GDR_GATE_SCALAR
    n_seq = (cu_seqlens.numel() - 1) if cu_seqlens is not None else B
    _need_contig(q, k, v, g, beta, S0, cu_seqlens)
    dev, th = _on_cuda(q), B * T * H
    _check(dev, ("k", k, q.dtype, th * d_k), ("v", v, q.dtype, th * d_v),
           ("g", g, torch.float32, th * (d_k if gate else 1)), ("beta", beta, torch.float32, th),
           ("S0", S0, torch.float32, n_seq * H * d_v * d_k), ("cu_seqlens", cu_seqlens, torch.int32, 1),
           ("out", out, q.dtype, th * d_v), ("S_final", S_final, torch.float32, n_seq * H * d_v * d_k))
    if out is None:
        out = torch.empty((B, T, H, d_v), dtype=q.dtype, device=q.device)
    if S_final is None and want_final:
        S_final = torch.empty((n_seq, H, d_v, d_k), dtype=torch.float32, device=q.device)
    ws_bytes = fwd_workspace_size(B, T, H, d_k, d_v, chunk, n_seq, cu_seqlens is not None, dtype,
                                  gate, path)
    if ws_bytes and (workspace is None or workspace.numel() * workspace.element_size() < ws_bytes):
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    ws_avail = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(dev, ("workspace", workspace, None, 0))
    st = _call_on(dev, lambda: lib().gdr_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(out), _ptr(S_final), B, T,
        H, d_k, d_v, chunk, _ptr(cu_seqlens), n_seq, dtype, gate, PATHS[path], _ptr(workspace),
        ws_avail, _stream(stream, dev)))
    if st != GDR_OK:
        raise GdrError(st, "gdr_fwd")
    return out, S_final


def gdr_fwd_product(q, k, v, g, beta, S0=None, *, chunk: int = 64, cu_seqlens=None, out=None,
                    S_final=None, want_final: bool = True, path: str = "auto", workspace=None,
                    stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Gated DeltaProduct prefill: k [B,T,n_h,H,d_k], v [B,T,n_h,H,d_v],
    beta [B,T,n_h,H]; returns (out [B,T,H,d_v], S_final)."""
    B, T, H, d_k = q.shape
    n_h = k.shape[2]
    d_v = v.shape[-1]
    dtype = _dtype_code(q)
    gate = GDR_GATE_PER_KEY_CHANNEL if g.dim() == 4 else GDR_GATE_SCALAR
    n_seq = (cu_seqlens.numel() - 1) if cu_seqlens is not None else B
    _need_contig(q, k, v, g, beta, S0, cu_seqlens)
    dev, th = _on_cuda(q), B * T * H
    _check(dev, ("k", k, q.dtype, th * n_h * d_k), ("v", v, q.dtype, th * n_h * d_v),
           ("g", g, torch.float32, th * (d_k if gate else 1)),
           ("beta", beta, torch.float32, th * n_h),
           ("S0", S0, torch.float32, n_seq * H * d_v * d_k), ("cu_seqlens", cu_seqlens, torch.int32, 1),
           ("out", out, q.dtype, th * d_v), ("S_final", S_final, torch.float32, n_seq * H * d_v * d_k))
    if out is None:
        out = torch.empty((B, T, H, d_v), dtype=q.dtype, device=q.device)
    if S_final is None and want_final:
        S_final = torch.empty((n_seq, H, d_v, d_k), dtype=torch.float32, device=q.device)
    ws_bytes = int(lib().gdr_fwd_product_workspace_size(B, T, H, n_h, d_k, d_v, chunk, n_seq,
                                                       int(cu_seqlens is not None), dtype, gate,
                                                       PATHS[path]))
    if ws_bytes and (workspace is None or workspace.numel() * workspace.element_size() < ws_bytes):
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    ws_avail = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(dev, ("workspace", workspace, None, 0))
    st = _call_on(dev, lambda: lib().gdr_fwd_product(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0), _ptr(out), _ptr(S_final), B, T,
        H, n_h, d_k, d_v, chunk, _ptr(cu_seqlens), n_seq, dtype, gate, PATHS[path],
        _ptr(workspace), ws_avail, _stream(stream, dev)))
    if st != GDR_OK:
        raise GdrError(st, "gdr_fwd_product")
    return out, S_final


def fwd_gdn2_workspace_size(B, T, H, d_k, d_v, chunk, n_seq, varlen, dtype, gate,
                            path="auto") -> int:
    return int(lib().gdr_fwd_gdn2_workspace_size(B, T, H, d_k, d_v, chunk, n_seq,
                                                 int(bool(varlen)), dtype, gate, PATHS[path]))


def gdr_fwd_gdn2(q, k, v, g, b, w, S0=None, *, chunk: int = 64, cu_seqlens=None, out=None,
                 S_final=None, want_final: bool = True, path: str = "auto", workspace=None,
                 stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Gated DeltaNet-2 prefill: erase gate b [B,T,H,d_k], write gate w
    [B,T,H,d_v] (fp32); returns (out [B,T,H,d_v], S_final)."""
    B, T, H, d_k = q.shape
    d_v = v.shape[-1]
    dtype = _dtype_code(q)
    gate = GDR_GATE_PER_KEY_CHANNEL if g.dim() == 4 else GDR_GATE_SCALAR
    n_seq = (cu_seqlens.numel() - 1) if cu_seqlens is not None else B
    _need_contig(q, k, v, g, b, w, S0, cu_seqlens)
    dev, th = _on_cuda(q), B * T * H
    _check(dev, ("k", k, q.dtype, th * d_k), ("v", v, q.dtype, th * d_v),
           ("g", g, torch.float32, th * (d_k if gate else 1)), ("b", b, torch.float32, th * d_k),
           ("w", w, torch.float32, th * d_v),
           ("S0", S0, torch.float32, n_seq * H * d_v * d_k), ("cu_seqlens", cu_seqlens, torch.int32, 1),
           ("out", out, q.dtype, th * d_v), ("S_final", S_final, torch.float32, n_seq * H * d_v * d_k))
    if out is None:
        out = torch.empty((B, T, H, d_v), dtype=q.dtype, device=q.device)
    if S_final is None and want_final:
        S_final = torch.empty((n_seq, H, d_v, d_k), dtype=torch.float32, device=q.device)
    ws_bytes = fwd_gdn2_workspace_size(B, T, H, d_k, d_v, chunk, n_seq, cu_seqlens is not None,
                                       dtype, gate, path)
    if ws_bytes and (workspace is None or workspace.numel() * workspace.element_size() < ws_bytes):
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    ws_avail = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(dev, ("workspace", workspace, None, 0))
    st = _call_on(dev, lambda: lib().gdr_fwd_gdn2(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), _ptr(S0), _ptr(out), _ptr(S_final),
        B, T, H, d_k, d_v, chunk, _ptr(cu_seqlens), n_seq, dtype, gate, PATHS[path],
        _ptr(workspace), ws_avail, _stream(stream, dev)))
    if st != GDR_OK:
        raise GdrError(st, "gdr_fwd_gdn2")
    return out, S_final


def gdr_decode_step_gdn2(q, k, v, g, b, w, S, *, out=None, stream=None) -> torch.Tensor:
    """Gated DeltaNet-2 decode of one token per sequence, updating ``S`` in place."""
    N, H, d_k = q.shape
    d_v = v.shape[-1]
    dtype = _dtype_code(q)
    gate = GDR_GATE_PER_KEY_CHANNEL if g.dim() == 3 else GDR_GATE_SCALAR
    _need_contig(q, k, v, g, b, w, S)
    dev, nh = _on_cuda(q), N * H
    _check(dev, ("k", k, q.dtype, nh * d_k), ("v", v, q.dtype, nh * d_v),
           ("g", g, torch.float32, nh * (d_k if gate else 1)), ("b", b, torch.float32, nh * d_k),
           ("w", w, torch.float32, nh * d_v), ("S", S, torch.float32, nh * d_v * d_k),
           ("out", out, q.dtype, nh * d_v))
    if out is None:
        out = torch.empty((N, H, d_v), dtype=q.dtype, device=q.device)
    st = _call_on(dev, lambda: lib().gdr_decode_step_gdn2(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b), _ptr(w), _ptr(S), _ptr(out), N, H, d_k, d_v,
        dtype, gate, _stream(stream, dev)))
    if st != GDR_OK:
        raise GdrError(st, "gdr_decode_step_gdn2")
    return out


def fwd_frame_workspace_size(B, T, H, d_k, d_v, n) -> int:
    return int(lib().gdr_fwd_frame_workspace_size(B, T, H, d_k, d_v, n))


def gdr_fwd_frame(q, k, v, g, gamma, n: int, S0=None, *, out=None, S_final=None,
                  want_final: bool = True, workspace=None,
                  stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Implicit frame-level update: frames of n tokens, gamma [B,T,H], g per
    frame [B,F,H] or [B,F,H,d_k]; returns (out [B,T,H,d_v], S_final [B,H,d_v,d_k])."""
    B, T, H, d_k = q.shape
    d_v = v.shape[-1]
    dtype = _dtype_code(q)
    gate = GDR_GATE_PER_KEY_CHANNEL if g.dim() == 4 else GDR_GATE_SCALAR
    _need_contig(q, k, v, g, gamma, S0)
    dev, th, F = _on_cuda(q), B * T * H, (T + n - 1) // max(n, 1)
    _check(dev, ("k", k, q.dtype, th * d_k), ("v", v, q.dtype, th * d_v),
           ("g", g, torch.float32, B * F * H * (d_k if gate else 1)),
           ("gamma", gamma, torch.float32, th), ("S0", S0, torch.float32, B * H * d_v * d_k),
           ("out", out, q.dtype, th * d_v), ("S_final", S_final, torch.float32, B * H * d_v * d_k))
    if out is None:
        out = torch.empty((B, T, H, d_v), dtype=q.dtype, device=q.device)
    if S_final is None and want_final:
        S_final = torch.empty((B, H, d_v, d_k), dtype=torch.float32, device=q.device)
    ws_bytes = fwd_frame_workspace_size(B, max(T, 1), H, d_k, d_v, n)
    if ws_bytes and (workspace is None or workspace.numel() * workspace.element_size() < ws_bytes):
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    ws_avail = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(dev, ("workspace", workspace, None, 0))
    st = _call_on(dev, lambda: lib().gdr_fwd_frame(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(gamma), _ptr(S0), _ptr(out), _ptr(S_final), B, T,
        H, d_k, d_v, n, dtype, gate, _ptr(workspace), ws_avail, _stream(stream, dev)))
    if st != GDR_OK:
        raise GdrError(st, "gdr_fwd_frame")
    return out, S_final


def gdr_decode_step(q, k, v, g, beta, S, *, out=None, stream=None) -> torch.Tensor:
    """Decode one token per sequence, updating ``S`` in place; returns out [N,H,d_v]."""
    N, H, d_k = q.shape
    d_v = v.shape[-1]
    dtype = _dtype_code(q)
    gate = GDR_GATE_PER_KEY_CHANNEL if g.dim() == 3 else GDR_GATE_SCALAR
    _need_contig(q, k, v, g, beta, S)
    dev, nh = _on_cuda(q), N * H
    _check(dev, ("k", k, q.dtype, nh * d_k), ("v", v, q.dtype, nh * d_v),
           ("g", g, torch.float32, nh * (d_k if gate else 1)), ("beta", beta, torch.float32, nh),
           ("S", S, torch.float32, nh * d_v * d_k), ("out", out, q.dtype, nh * d_v))
    if out is None:
        out = torch.empty((N, H, d_v), dtype=q.dtype, device=q.device)
    st = _call_on(dev, lambda: lib().gdr_decode_step(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S), _ptr(out), N, H, d_k, d_v, dtype,
        gate, _stream(stream, dev)))
    if st != GDR_OK:
        raise GdrError(st, "gdr_decode_step")
    return out


def device_status(stream=None) -> int:
    return int(lib().gdr_device_status(_stream(stream)))


def selftest_wait_timeout(spin_limit: int, stream=None) -> int:
    return int(lib().gdr_selftest_wait_timeout(spin_limit, _stream(stream)))


def checked_build() -> bool:
    """True when the loaded library is the checked build (gdr.h, gdr_checked_build)."""
    return bool(lib().gdr_checked_build())


def selftest_bounds(stream=None) -> int:
    return int(lib().gdr_selftest_bounds(_stream(stream)))


def set_gram_spread_limit(limit: float) -> float:
    """Set the tensor-core prefill's Gram range limit (gdr.h,
    gdr_set_gram_spread_limit); returns the previous one."""
    return float(lib().gdr_set_gram_spread_limit(float(limit)))


def profile_enable(on: bool = True) -> None:
    lib().gdr_profile_enable(1 if on else 0)


def profile_read() -> dict:
    """{kernel: (launches, total_ms)} since the previous read (then reset)."""
    res = {}
    for name, kid in KERNELS.items():
        n = ctypes.c_longlong(0)
        ms = ctypes.c_double(0.0)
        st = lib().gdr_profile_read(kid, ctypes.byref(n), ctypes.byref(ms))
        if st != GDR_OK:
            raise GdrError(st, "gdr_profile_read")
        res[name] = (int(n.value), float(ms.value))
    return res
