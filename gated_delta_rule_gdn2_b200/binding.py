"""Thin ctypes binding of libgdn2.so (argument marshalling only).

The ``gdn2_*`` functions mirror the C entry points of include/gdn2.h one to one:
tensor arguments may be torch tensors (their ``data_ptr()`` is passed), plain
integers (raw device addresses) or None (a null pointer).  ``chunk_fwd``,
``decode_step`` and ``chunk_bwd`` are conveniences that check shapes, allocate
the outputs and the workspace with torch on the inputs' device and raise
``Gdn2Error`` on a non-zero status.  Every step of the computation runs in the
library's CUDA kernels; there is no other code path.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libgdn2.so")

GDN2_BF16 = 0
GDN2_FP32 = 1
STATUS = {0: "GDN2_OK", -1: "GDN2_ERR_INVALID_ARG", -2: "GDN2_ERR_UNSUPPORTED", -3: "GDN2_ERR_CUDA",
          -4: "GDN2_ERR_TIMEOUT", -5: "GDN2_ERR_WORKSPACE"}

# name -> (restype, argtypes)
_P, _I, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "gdn2_version": (_I, []),
    "gdn2_status_string": (ctypes.c_char_p, [_I]),
    "gdn2_get_device_status": (_I, [_P]),
    "gdn2_chunk_fwd_workspace": (_Z, [_I] * 6),
    "gdn2_chunk_fwd": (_I, [_P] * 9 + [_I] * 6 + [_P, _Z, _P]),
    "gdn2_decode_step": (_I, [_P] * 8 + [_I] * 5 + [_P]),
    "gdn2_chunk_bwd_workspace": (_Z, [_I] * 6),
    "gdn2_chunk_bwd": (_I, [_P] * 16 + [_I] * 6 + [_P, _Z, _P]),
    "gdn2_chunk_fwd_noalloc": (_I, [_P] * 9 + [_I] * 6 + [_P]),
    "gdn2_chunk_states_bytes": (_Z, [_I] * 6),
    "gdn2_chunk_fwd_save": (_I, [_P] * 10 + [_I] * 6 + [_P, _Z, _P]),
    "gdn2_chunk_bwd_saved_workspace": (_Z, [_I] * 6),
    "gdn2_chunk_bwd_saved": (_I, [_P] * 17 + [_I] * 6 + [_P, _Z, _P]),
}

_lib = None


class Gdn2Error(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__("%s failed: %s (%d)" % (what, STATUS.get(status, "unknown"), status))


def load() -> ctypes.CDLL:
    """Load the in-tree libgdn2.so.  Raises if it has not been built: there is
    no fallback implementation."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libgdn2.so is not built (%s); run "
                              "`python -m gated_delta_rule_gdn2_b200.build`" % LIB_PATH)
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# --------------------------------------------------------------------------
# one-to-one C entry points


def gdn2_version() -> int:
    return load().gdn2_version()


def gdn2_status_string(status: int) -> str:
    return load().gdn2_status_string(status).decode()


def gdn2_get_device_status(stream=None) -> int:
    return load().gdn2_get_device_status(_stream(stream))


def gdn2_chunk_fwd_workspace(B, T, H, dk, dv, dtype) -> int:
    return load().gdn2_chunk_fwd_workspace(B, T, H, dk, dv, dtype)


def gdn2_chunk_bwd_workspace(B, T, H, dk, dv, dtype) -> int:
    return load().gdn2_chunk_bwd_workspace(B, T, H, dk, dv, dtype)


def gdn2_chunk_fwd(q, k, v, log_alpha, b, w, S0, o, S_T, B, T, H, dk, dv, dtype, ws, ws_bytes,
                   stream=None) -> int:
    return load().gdn2_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w),
                                 _ptr(S0), _ptr(o), _ptr(S_T), B, T, H, dk, dv, dtype, _ptr(ws),
                                 ws_bytes, _stream(stream))


def gdn2_chunk_fwd_noalloc(q, k, v, log_alpha, b, w, S0, o, S_T, B, T, H, dk, dv, dtype,
                           stream=None) -> int:
    """gdn2_chunk_fwd for callers that cannot allocate: the scratch comes from
    a fixed 8 MiB array inside the library (see include/gdn2.h)."""
    return load().gdn2_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w),
                                         _ptr(S0), _ptr(o), _ptr(S_T), B, T, H, dk, dv, dtype,
                                         _stream(stream))


def gdn2_chunk_states_bytes(B, T, H, dk, dv, dtype) -> int:
    return load().gdn2_chunk_states_bytes(B, T, H, dk, dv, dtype)


def gdn2_chunk_bwd_saved_workspace(B, T, H, dk, dv, dtype) -> int:
    return load().gdn2_chunk_bwd_saved_workspace(B, T, H, dk, dv, dtype)


def gdn2_chunk_fwd_save(q, k, v, log_alpha, b, w, S0, o, S_T, states, B, T, H, dk, dv, dtype, ws, ws_bytes,
                        stream=None) -> int:
    return load().gdn2_chunk_fwd_save(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w),
                                      _ptr(S0), _ptr(o), _ptr(S_T), _ptr(states), B, T, H, dk, dv, dtype,
                                      _ptr(ws), ws_bytes, _stream(stream))


def gdn2_chunk_bwd_saved(q, k, v, log_alpha, b, w, S0, dO, dS_T, states, dq, dk_, dv_, dlog_alpha, db, dw,
                         dS0, B, T, H, dk, dv, dtype, ws, ws_bytes, stream=None) -> int:
    return load().gdn2_chunk_bwd_saved(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w),
                                       _ptr(S0), _ptr(dO), _ptr(dS_T), _ptr(states), _ptr(dq), _ptr(dk_),
                                       _ptr(dv_), _ptr(dlog_alpha), _ptr(db), _ptr(dw), _ptr(dS0), B, T, H,
                                       dk, dv, dtype, _ptr(ws), ws_bytes, _stream(stream))


def gdn2_decode_step(q, k, v, log_alpha, b, w, S, o, B, H, dk, dv, dtype, stream=None) -> int:
    return load().gdn2_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w),
                                   _ptr(S), _ptr(o), B, H, dk, dv, dtype, _stream(stream))


def gdn2_chunk_bwd(q, k, v, log_alpha, b, w, S0, dO, dS_T, dq, dk_, dv_, dlog_alpha, db, dw, dS0,
                   B, T, H, dk, dv, dtype, ws, ws_bytes, stream=None) -> int:
    return load().gdn2_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w),
                                 _ptr(S0), _ptr(dO), _ptr(dS_T), _ptr(dq), _ptr(dk_), _ptr(dv_),
                                 _ptr(dlog_alpha), _ptr(db), _ptr(dw), _ptr(dS0), B, T, H, dk, dv,
                                 dtype, _ptr(ws), ws_bytes, _stream(stream))


# --------------------------------------------------------------------------
# torch conveniences


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return GDN2_BF16
    if t.dtype == torch.float32:
        return GDN2_FP32
    raise TypeError("token tensors must be bfloat16 or float32, got %s" % t.dtype)


def _check_tokens(q, k, v, log_alpha, b, w, lead_dims):
    dt = q.dtype
    for name, t in (("q", q), ("k", k), ("v", v), ("log_alpha", log_alpha), ("b", b), ("w", w)):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != dt:
            raise ValueError("%s must be a contiguous CUDA tensor of dtype %s" % (name, dt))
    lead = tuple(q.shape[:lead_dims])
    for t in (k, log_alpha, b):
        if tuple(t.shape) != tuple(q.shape):
            raise ValueError("q, k, log_alpha and b must share a shape")
    if tuple(w.shape) != tuple(v.shape) or tuple(v.shape[:lead_dims]) != lead:
        raise ValueError("v and w must be %s + (dv,)" % (lead,))


def _raise(st, what):
    if st != 0:
        raise Gdn2Error(st, what)


def chunk_fwd(q, k, v, log_alpha, b, w, S0=None, output_final_state=True, save_states=False, stream=None):
    """o, S_T = chunk_fwd(...) for token tensors [B,T,H,D] (bf16 or fp32).

    With save_states=True returns (o, S_T, states): the chunk-boundary states
    for chunk_bwd(..., states=states)."""
    import torch
    _check_tokens(q, k, v, log_alpha, b, w, 3)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device) if output_final_state else None
    nws = gdn2_chunk_fwd_workspace(B, T, H, dk, dv, dt)
    ws = torch.empty(nws, dtype=torch.uint8, device=q.device) if nws else None
    if not save_states:
        _raise(gdn2_chunk_fwd(q, k, v, log_alpha, b, w, S0, o, S_T, B, T, H, dk, dv, dt, ws, nws, stream),
               "gdn2_chunk_fwd")
        return o, S_T
    nst = gdn2_chunk_states_bytes(B, T, H, dk, dv, dt)
    states = torch.empty(nst, dtype=torch.uint8, device=q.device) if nst else None
    _raise(gdn2_chunk_fwd_save(q, k, v, log_alpha, b, w, S0, o, S_T, states, B, T, H, dk, dv, dt, ws, nws,
                               stream), "gdn2_chunk_fwd_save")
    return o, S_T, states


def decode_step(q, k, v, log_alpha, b, w, S, stream=None):
    """o = decode_step(...): tokens [B,H,D]; S [B,H,dk,dv] fp32 updated in place."""
    import torch
    _check_tokens(q, k, v, log_alpha, b, w, 2)
    B, H, dk = q.shape
    dv = v.shape[-1]
    if S.dtype != torch.float32 or tuple(S.shape) != (B, H, dk, dv) or not S.is_contiguous():
        raise ValueError("S must be a contiguous fp32 tensor of shape %s" % ((B, H, dk, dv),))
    o = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    _raise(gdn2_decode_step(q, k, v, log_alpha, b, w, S, o, B, H, dk, dv, _dtype_code(q), stream),
           "gdn2_decode_step")
    return o


def chunk_bwd(q, k, v, log_alpha, b, w, S0, dO, dS_T=None, need_dS0=True, states=None, stream=None):
    """Gradients (dq, dk, dv, dlog_alpha, db, dw, dS0) of gdn2_chunk_fwd.

    `states` from chunk_fwd(..., save_states=True) skips the state recompute."""
    import torch
    _check_tokens(q, k, v, log_alpha, b, w, 3)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    g = {n: torch.empty_like(q) for n in ("dq", "dk", "dlog_alpha", "db")}
    g.update({n: torch.empty_like(v) for n in ("dv", "dw")})
    g["dS0"] = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device) if need_dS0 else None
    if states is None:
        nws = gdn2_chunk_bwd_workspace(B, T, H, dk, dv, dt)
        ws = torch.empty(nws, dtype=torch.uint8, device=q.device) if nws else None
        _raise(gdn2_chunk_bwd(q, k, v, log_alpha, b, w, S0, dO, dS_T, g["dq"], g["dk"], g["dv"],
                              g["dlog_alpha"], g["db"], g["dw"], g["dS0"], B, T, H, dk, dv, dt, ws, nws,
                              stream), "gdn2_chunk_bwd")
        return g
    nws = gdn2_chunk_bwd_saved_workspace(B, T, H, dk, dv, dt)
    ws = torch.empty(nws, dtype=torch.uint8, device=q.device) if nws else None
    _raise(gdn2_chunk_bwd_saved(q, k, v, log_alpha, b, w, S0, dO, dS_T, states, g["dq"], g["dk"], g["dv"],
                                g["dlog_alpha"], g["db"], g["dw"], g["dS0"], B, T, H, dk, dv, dt, ws, nws,
                                stream), "gdn2_chunk_bwd_saved")
    return g
