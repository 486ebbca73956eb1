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
    "gdn2_debug_set": (_I, [_I, ctypes.c_longlong]),
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
    "gdn2_chunk_fwd_varlen_workspace": (_Z, [_I] * 6),
    "gdn2_chunk_fwd_varlen": (_I, [_P] * 10 + [_I] * 6 + [_P, _Z, _P]),
    "gdn2_chunk_bwd_varlen_workspace": (_Z, [_I] * 6),
    "gdn2_chunk_bwd_varlen": (_I, [_P] * 17 + [_I] * 6 + [_P, _Z, _P]),
    "gdn2_chunk_states_varlen_bytes": (_Z, [_I] * 6),
    "gdn2_chunk_fwd_save_varlen": (_I, [_P] * 11 + [_I] * 6 + [_P, _Z, _P]),
    "gdn2_chunk_bwd_saved_varlen_workspace": (_Z, [_I] * 6),
    "gdn2_chunk_bwd_saved_varlen": (_I, [_P] * 18 + [_I] * 6 + [_P, _Z, _P]),
    "gdn2_chunk_fwd_kda": (_I, [_P] * 8 + [_I] * 6 + [_P, _Z, _P]),
    "gdn2_chunk_fwd_gdn": (_I, [_P] * 8 + [_I] * 6 + [_P, _Z, _P]),
    "gdn2_chunk_bwd_kda": (_I, [_P] * 14 + [_I] * 6 + [_P, _Z, _P]),
    "gdn2_chunk_bwd_gdn": (_I, [_P] * 14 + [_I] * 6 + [_P, _Z, _P]),
    "gdn2_decode_step_kda": (_I, [_P] * 7 + [_I] * 5 + [_P]),
    "gdn2_decode_step_gdn": (_I, [_P] * 7 + [_I] * 5 + [_P]),
    "gdn2_chunk_fwd_gated": (_I, [_P] * 11 + [_I] * 6 + [_P, _Z, _P]),
    "gdn2_prologue_fwd": (_I, [_P] * 6 + [_I] + [_P] * 9 + [_P] + [_I] * 6 + [_P]),
    "gdn2_prologue_bwd_workspace": (_Z, [_I] * 7),
    "gdn2_prologue_bwd": (_I, [_P] * 6 + [_I] + [_P] * 18 + [_P] + [_I] * 6 + [_P, _Z, _P]),
    "gdn2_output_gate_fwd": (_I, [_P] * 4 + [ctypes.c_longlong, _I, _I, _I, _P]),
    "gdn2_output_gate_bwd_workspace": (_Z, [ctypes.c_longlong, _I, _I]),
    "gdn2_output_gate_bwd": (_I, [_P] * 7 + [ctypes.c_longlong, _I, _I, _I, _P, _Z, _P]),
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


GDN2_DEBUG_WAIT_LIMIT = 0
GDN2_DEBUG_WITHHOLD_READY = 1


def gdn2_debug_set(knob: int, value: int) -> int:
    return load().gdn2_debug_set(knob, value)


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


def gdn2_chunk_fwd_varlen_workspace(N, total_T, H, dk, dv, dtype) -> int:
    return load().gdn2_chunk_fwd_varlen_workspace(N, total_T, H, dk, dv, dtype)


def gdn2_chunk_fwd_varlen(q, k, v, log_alpha, b, w, S0, o, S_T, cu_seqlens, N, total_T, H, dk, dv, dtype, ws,
                          ws_bytes, stream=None) -> int:
    return load().gdn2_chunk_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(S0),
                                        _ptr(o), _ptr(S_T), _ptr(cu_seqlens), N, total_T, H, dk, dv, dtype,
                                        _ptr(ws), ws_bytes, _stream(stream))


def gdn2_chunk_bwd_varlen_workspace(N, total_T, H, dk, dv, dtype) -> int:
    return load().gdn2_chunk_bwd_varlen_workspace(N, total_T, H, dk, dv, dtype)


def gdn2_chunk_bwd_varlen(q, k, v, log_alpha, b, w, S0, dO, dS_T, dq, dk_, dv_, dlog_alpha, db, dw, dS0,
                          cu_seqlens, N, total_T, H, dk, dv, dtype, ws, ws_bytes, stream=None) -> int:
    return load().gdn2_chunk_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(S0),
                                        _ptr(dO), _ptr(dS_T), _ptr(dq), _ptr(dk_), _ptr(dv_), _ptr(dlog_alpha),
                                        _ptr(db), _ptr(dw), _ptr(dS0), _ptr(cu_seqlens), N, total_T, H, dk, dv,
                                        dtype, _ptr(ws), ws_bytes, _stream(stream))


def gdn2_chunk_states_varlen_bytes(N, total_T, H, dk, dv, dtype) -> int:
    return load().gdn2_chunk_states_varlen_bytes(N, total_T, H, dk, dv, dtype)


def gdn2_chunk_fwd_save_varlen(q, k, v, log_alpha, b, w, S0, o, S_T, states, cu_seqlens, N, total_T, H, dk, dv,
                               dtype, ws, ws_bytes, stream=None) -> int:
    return load().gdn2_chunk_fwd_save_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w),
                                             _ptr(S0), _ptr(o), _ptr(S_T), _ptr(states), _ptr(cu_seqlens), N,
                                             total_T, H, dk, dv, dtype, _ptr(ws), ws_bytes, _stream(stream))


def gdn2_chunk_bwd_saved_varlen_workspace(N, total_T, H, dk, dv, dtype) -> int:
    return load().gdn2_chunk_bwd_saved_varlen_workspace(N, total_T, H, dk, dv, dtype)


def gdn2_chunk_bwd_saved_varlen(q, k, v, log_alpha, b, w, S0, dO, dS_T, states, dq, dk_, dv_, dlog_alpha, db, dw,
                                dS0, cu_seqlens, N, total_T, H, dk, dv, dtype, ws, ws_bytes, stream=None) -> int:
    return load().gdn2_chunk_bwd_saved_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w),
                                              _ptr(S0), _ptr(dO), _ptr(dS_T), _ptr(states), _ptr(dq), _ptr(dk_),
                                              _ptr(dv_), _ptr(dlog_alpha), _ptr(db), _ptr(dw), _ptr(dS0),
                                              _ptr(cu_seqlens), N, total_T, H, dk, dv, dtype, _ptr(ws), ws_bytes,
                                              _stream(stream))


def _reduced(name):
    def fwd(q, k, v, log_alpha, beta, S0, o, S_T, B, T, H, dk, dv, dtype, ws, ws_bytes, stream=None):
        return getattr(load(), name)(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0), _ptr(o),
                                     _ptr(S_T), B, T, H, dk, dv, dtype, _ptr(ws), ws_bytes, _stream(stream))

    def bwd(q, k, v, log_alpha, beta, S0, dO, dS_T, dq, dk_, dv_, dlog_alpha, dbeta, dS0, B, T, H, dk, dv, dtype,
            ws, ws_bytes, stream=None):
        return getattr(load(), name)(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S0), _ptr(dO),
                                     _ptr(dS_T), _ptr(dq), _ptr(dk_), _ptr(dv_), _ptr(dlog_alpha), _ptr(dbeta),
                                     _ptr(dS0), B, T, H, dk, dv, dtype, _ptr(ws), ws_bytes, _stream(stream))

    def dec(q, k, v, log_alpha, beta, S, o, B, H, dk, dv, dtype, stream=None):
        return getattr(load(), name)(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(S), _ptr(o),
                                     B, H, dk, dv, dtype, _stream(stream))

    f = {"fwd": fwd, "bwd": bwd, "dec": dec}[name.split("_")[2][:3] if "decode" not in name else "dec"]
    f.__name__ = name
    f.__doc__ = "%s of include/gdn2.h (reduced gates: one scalar beta per token and head)." % name
    return f


gdn2_chunk_fwd_kda = _reduced("gdn2_chunk_fwd_kda")
gdn2_chunk_fwd_gdn = _reduced("gdn2_chunk_fwd_gdn")
gdn2_chunk_bwd_kda = _reduced("gdn2_chunk_bwd_kda")
gdn2_chunk_bwd_gdn = _reduced("gdn2_chunk_bwd_gdn")
gdn2_decode_step_kda = _reduced("gdn2_decode_step_kda")
gdn2_decode_step_gdn = _reduced("gdn2_decode_step_gdn")


def gdn2_prologue_fwd(xq, xk, xv, Wq, Wk, Wv, K, xa, xb, xw, q, k, v, log_alpha, b, w, cu_seqlens, B, T, H, dk,
                      dv, dtype, stream=None) -> int:
    return load().gdn2_prologue_fwd(*[_ptr(t) for t in (xq, xk, xv, Wq, Wk, Wv)], K,
                                    *[_ptr(t) for t in (xa, xb, xw, q, k, v, log_alpha, b, w, cu_seqlens)],
                                    B, T, H, dk, dv, dtype, _stream(stream))


def gdn2_prologue_bwd_workspace(B, T, H, dk, dv, K, packed) -> int:
    return load().gdn2_prologue_bwd_workspace(B, T, H, dk, dv, K, int(bool(packed)))


def gdn2_prologue_bwd(xq, xk, xv, Wq, Wk, Wv, K, xa, xb, xw, dq, dk_, dv_, dlog_alpha, db, dw, dxq, dxk, dxv, dWq,
                      dWk, dWv, dxa, dxb, dxw, cu_seqlens, B, T, H, dk, dv, dtype, ws, ws_bytes, stream=None) -> int:
    return load().gdn2_prologue_bwd(*[_ptr(t) for t in (xq, xk, xv, Wq, Wk, Wv)], K,
                                    *[_ptr(t) for t in (xa, xb, xw, dq, dk_, dv_, dlog_alpha, db, dw, dxq, dxk, dxv,
                                                        dWq, dWk, dWv, dxa, dxb, dxw, cu_seqlens)],
                                    B, T, H, dk, dv, dtype, _ptr(ws), ws_bytes, _stream(stream))


def gdn2_chunk_fwd_gated(q, k, v, log_alpha, b, w, S0, g, gamma, z, S_T, B, T, H, dk, dv, dtype, ws, ws_bytes,
                         stream=None) -> int:
    return load().gdn2_chunk_fwd_gated(*[_ptr(t) for t in (q, k, v, log_alpha, b, w, S0, g, gamma, z, S_T)], B, T, H,
                                       dk, dv, dtype, _ptr(ws), ws_bytes, _stream(stream))


def gdn2_output_gate_fwd(o, g, gamma, z, rows, H, dv, dtype, stream=None) -> int:
    return load().gdn2_output_gate_fwd(_ptr(o), _ptr(g), _ptr(gamma), _ptr(z), rows, H, dv, dtype, _stream(stream))


def gdn2_output_gate_bwd_workspace(rows, H, dv) -> int:
    return load().gdn2_output_gate_bwd_workspace(rows, H, dv)


def gdn2_output_gate_bwd(o, g, gamma, dz, dO, dg, dgamma, rows, H, dv, dtype, ws, ws_bytes, stream=None) -> int:
    return load().gdn2_output_gate_bwd(_ptr(o), _ptr(g), _ptr(gamma), _ptr(dz), _ptr(dO), _ptr(dg), _ptr(dgamma),
                                       rows, H, dv, dtype, _ptr(ws), ws_bytes, _stream(stream))


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


def _check_cu(cu_seqlens, total_T):
    import torch
    if not cu_seqlens.is_cuda or cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or \
            not cu_seqlens.is_contiguous() or cu_seqlens.numel() < 1:
        raise ValueError("cu_seqlens must be a contiguous 1-D int32 CUDA tensor of N + 1 offsets")
    return cu_seqlens.numel() - 1


def chunk_fwd_varlen(q, k, v, log_alpha, b, w, cu_seqlens, S0=None, output_final_state=True, save_states=False,
                     stream=None):
    """o, S_T = chunk_fwd_varlen(...) for packed token tensors [total_T, H, D]
    (or [1, total_T, H, D]) holding N sequences delimited by cu_seqlens (N + 1
    int32 offsets on the device).  S0 / S_T are [N, H, dk, dv].  With
    save_states=True returns (o, S_T, states) for chunk_bwd_varlen."""
    import torch
    q, k, v, log_alpha, b, w = (t.reshape(t.shape[-3:]) if t.dim() == 4 else t for t in (q, k, v, log_alpha, b, w))
    _check_tokens(q, k, v, log_alpha, b, w, 2)
    T, H, dk = q.shape
    dv = v.shape[-1]
    N = _check_cu(cu_seqlens, T)
    dt = _dtype_code(q)
    o = torch.empty((T, H, dv), dtype=q.dtype, device=q.device)
    S_T = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device) if output_final_state else None
    nws = gdn2_chunk_fwd_varlen_workspace(N, T, H, dk, dv, dt)
    ws = torch.empty(nws, dtype=torch.uint8, device=q.device) if nws else None
    if not save_states:
        _raise(gdn2_chunk_fwd_varlen(q, k, v, log_alpha, b, w, S0, o, S_T, cu_seqlens, N, T, H, dk, dv, dt, ws, nws,
                                     stream), "gdn2_chunk_fwd_varlen")
        return o, S_T
    nst = gdn2_chunk_states_varlen_bytes(N, T, H, dk, dv, dt)
    states = torch.empty(nst, dtype=torch.uint8, device=q.device) if nst else None
    _raise(gdn2_chunk_fwd_save_varlen(q, k, v, log_alpha, b, w, S0, o, S_T, states, cu_seqlens, N, T, H, dk, dv, dt,
                                      ws, nws, stream), "gdn2_chunk_fwd_save_varlen")
    return o, S_T, states


def chunk_bwd_varlen(q, k, v, log_alpha, b, w, cu_seqlens, S0, dO, dS_T=None, need_dS0=True, states=None,
                     stream=None):
    """Gradients of chunk_fwd_varlen: dq, dk, dv, dlog_alpha, db, dw as [total_T, H, D], dS0 [N, H, dk, dv]."""
    import torch
    q, k, v, log_alpha, b, w, dO = (t.reshape(t.shape[-3:]) if t.dim() == 4 else t
                                    for t in (q, k, v, log_alpha, b, w, dO))
    _check_tokens(q, k, v, log_alpha, b, w, 2)
    T, H, dk = q.shape
    dv = v.shape[-1]
    N = _check_cu(cu_seqlens, T)
    dt = _dtype_code(q)
    g = {n: torch.empty_like(q) for n in ("dq", "dk", "dlog_alpha", "db")}
    g.update({n: torch.empty_like(v) for n in ("dv", "dw")})
    g["dS0"] = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device) if need_dS0 else None
    if states is None:
        nws = gdn2_chunk_bwd_varlen_workspace(N, T, H, dk, dv, dt)
        ws = torch.empty(nws, dtype=torch.uint8, device=q.device) if nws else None
        _raise(gdn2_chunk_bwd_varlen(q, k, v, log_alpha, b, w, S0, dO, dS_T, g["dq"], g["dk"], g["dv"],
                                     g["dlog_alpha"], g["db"], g["dw"], g["dS0"], cu_seqlens, N, T, H, dk, dv, dt,
                                     ws, nws, stream), "gdn2_chunk_bwd_varlen")
        return g
    nws = gdn2_chunk_bwd_saved_varlen_workspace(N, T, H, dk, dv, dt)
    ws = torch.empty(nws, dtype=torch.uint8, device=q.device) if nws else None
    _raise(gdn2_chunk_bwd_saved_varlen(q, k, v, log_alpha, b, w, S0, dO, dS_T, states, g["dq"], g["dk"], g["dv"],
                                       g["dlog_alpha"], g["db"], g["dw"], g["dS0"], cu_seqlens, N, T, H, dk, dv,
                                       dt, ws, nws, stream), "gdn2_chunk_bwd_saved_varlen")
    return g


def _check_reduced(q, k, v, log_alpha, beta, mode, lead_dims):
    if mode not in ("kda", "gdn"):
        raise ValueError("mode must be 'kda' or 'gdn'")
    lead = tuple(q.shape[:lead_dims])
    for name, t in (("q", q), ("k", k), ("v", v), ("log_alpha", log_alpha), ("beta", beta)):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != q.dtype:
            raise ValueError("%s must be a contiguous CUDA tensor of dtype %s" % (name, q.dtype))
    want_la = q.shape if mode == "kda" else lead
    if tuple(k.shape) != tuple(q.shape) or tuple(log_alpha.shape) != tuple(want_la) or tuple(beta.shape) != lead \
            or tuple(v.shape[:lead_dims]) != lead:
        raise ValueError("shapes: q, k %s; log_alpha %s; beta %s" % (tuple(q.shape), tuple(want_la), lead))


def chunk_fwd_reduced(q, k, v, log_alpha, beta, mode="kda", S0=None, output_final_state=True, stream=None):
    """o, S_T with reduced gates: mode 'kda' (beta [B,T,H] for both gates,
    log_alpha [B,T,H,dk]) or 'gdn' (also a scalar decay, log_alpha [B,T,H])."""
    import torch
    _check_reduced(q, k, v, log_alpha, beta, mode, 3)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device) if output_final_state else None
    nws = gdn2_chunk_fwd_workspace(B, T, H, dk, dv, dt)
    ws = torch.empty(nws, dtype=torch.uint8, device=q.device) if nws else None
    fn = gdn2_chunk_fwd_kda if mode == "kda" else gdn2_chunk_fwd_gdn
    _raise(fn(q, k, v, log_alpha, beta, S0, o, S_T, B, T, H, dk, dv, dt, ws, nws, stream), fn.__name__)
    return o, S_T


def chunk_bwd_reduced(q, k, v, log_alpha, beta, S0, dO, dS_T=None, mode="kda", need_dS0=True, stream=None):
    """Gradients with reduced gates: dq, dk, dv, dlog_alpha (the shape of
    log_alpha), dbeta [B,T,H] and dS0."""
    import torch
    _check_reduced(q, k, v, log_alpha, beta, mode, 3)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    g = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
         "dlog_alpha": torch.empty_like(log_alpha), "dbeta": torch.empty_like(beta),
         "dS0": torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device) if need_dS0 else None}
    nws = gdn2_chunk_bwd_workspace(B, T, H, dk, dv, dt)
    ws = torch.empty(nws, dtype=torch.uint8, device=q.device) if nws else None
    fn = gdn2_chunk_bwd_kda if mode == "kda" else gdn2_chunk_bwd_gdn
    _raise(fn(q, k, v, log_alpha, beta, S0, dO, dS_T, g["dq"], g["dk"], g["dv"], g["dlog_alpha"], g["dbeta"],
              g["dS0"], B, T, H, dk, dv, dt, ws, nws, stream), fn.__name__)
    return g


def decode_step_reduced(q, k, v, log_alpha, beta, S, mode="kda", stream=None):
    """o = one decode step with reduced gates (beta [B,H]; 'gdn': log_alpha [B,H]); S updated in place."""
    import torch
    _check_reduced(q, k, v, log_alpha, beta, mode, 2)
    B, H, dk = q.shape
    dv = v.shape[-1]
    o = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    fn = gdn2_decode_step_kda if mode == "kda" else gdn2_decode_step_gdn
    _raise(fn(q, k, v, log_alpha, beta, S, o, B, H, dk, dv, _dtype_code(q), stream), fn.__name__)
    return o


def prologue(xq, xk, xv, Wq, Wk, Wv, xa, xb, xw, cu_seqlens=None, stream=None):
    """The mixer's inputs (q, k, v, log_alpha, b, w) from the projections and
    gate pre-activations: token tensors [B, T, H, D] (or packed [T, H, D] with
    cu_seqlens), filters fp32 [H*D, K]."""
    import torch
    packed = cu_seqlens is not None
    H, dk = xq.shape[-2], xq.shape[-1]
    dv = xv.shape[-1]
    B, T = (cu_seqlens.numel() - 1, xq.shape[0]) if packed else (xq.shape[0], xq.shape[1])
    K = Wq.shape[-1]
    outs = [torch.empty_like(t) for t in (xq, xk, xv, xa, xb, xw)]
    _raise(gdn2_prologue_fwd(xq, xk, xv, Wq, Wk, Wv, K, xa, xb, xw, *outs, cu_seqlens, B, T, H, dk, dv,
                             _dtype_code(xq), stream), "gdn2_prologue_fwd")
    return dict(zip(("q", "k", "v", "log_alpha", "b", "w"), outs))


def prologue_bwd(xq, xk, xv, Wq, Wk, Wv, xa, xb, xw, grads, cu_seqlens=None, stream=None):
    """Gradients of the prologue's inputs from `grads` (dq, dk, dv, dlog_alpha, db, dw)."""
    import torch
    packed = cu_seqlens is not None
    H, dk = xq.shape[-2], xq.shape[-1]
    dv = xv.shape[-1]
    B, T = (cu_seqlens.numel() - 1, xq.shape[0]) if packed else (xq.shape[0], xq.shape[1])
    K = Wq.shape[-1]
    dx = {n: torch.empty_like(t) for n, t in (("dxq", xq), ("dxk", xk), ("dxv", xv), ("dxa", xa), ("dxb", xb),
                                             ("dxw", xw))}
    dW = {n: torch.empty_like(t) for n, t in (("dWq", Wq), ("dWk", Wk), ("dWv", Wv))}
    nws = gdn2_prologue_bwd_workspace(B, T, H, dk, dv, K, packed)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=xq.device)
    _raise(gdn2_prologue_bwd(xq, xk, xv, Wq, Wk, Wv, K, xa, xb, xw, grads["dq"], grads["dk"], grads["dv"],
                             grads["dlog_alpha"], grads["db"], grads["dw"], dx["dxq"], dx["dxk"], dx["dxv"],
                             dW["dWq"], dW["dWk"], dW["dWv"], dx["dxa"], dx["dxb"], dx["dxw"], cu_seqlens, B, T, H,
                             dk, dv, _dtype_code(xq), ws, nws, stream), "gdn2_prologue_bwd")
    dx.update(dW)
    return dx


def output_gate(o, g, gamma, stream=None):
    """z = o / rms(o) * gamma * silu(g) per token and head (o, g [..., H, dv], gamma fp32 [dv])."""
    import torch
    H, dv = o.shape[-2], o.shape[-1]
    rows = o.numel() // (H * dv)
    z = torch.empty_like(o)
    _raise(gdn2_output_gate_fwd(o, g, gamma, z, rows, H, dv, _dtype_code(o), stream), "gdn2_output_gate_fwd")
    return z


def output_gate_bwd(o, g, gamma, dz, stream=None):
    """(do, dg, dgamma) of output_gate."""
    import torch
    H, dv = o.shape[-2], o.shape[-1]
    rows = o.numel() // (H * dv)
    dO, dg, dgamma = torch.empty_like(o), torch.empty_like(g), torch.empty_like(gamma)
    nws = gdn2_output_gate_bwd_workspace(rows, H, dv)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=o.device)
    _raise(gdn2_output_gate_bwd(o, g, gamma, dz, dO, dg, dgamma, rows, H, dv, _dtype_code(o), ws, nws, stream),
           "gdn2_output_gate_bwd")
    return dO, dg, dgamma


def chunk_fwd_gated(q, k, v, log_alpha, b, w, g, gamma, S0=None, output_final_state=True, stream=None):
    """z, S_T: the forward with the output epilogue z = o / rms(o) * gamma * silu(g)."""
    import torch
    _check_tokens(q, k, v, log_alpha, b, w, 3)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    z = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device) if output_final_state else None
    nws = gdn2_chunk_fwd_workspace(B, T, H, dk, dv, dt)
    ws = torch.empty(nws, dtype=torch.uint8, device=q.device) if nws else None
    _raise(gdn2_chunk_fwd_gated(q, k, v, log_alpha, b, w, S0, g, gamma, z, S_T, B, T, H, dk, dv, dt, ws, nws,
                                stream), "gdn2_chunk_fwd_gated")
    return z, S_T
