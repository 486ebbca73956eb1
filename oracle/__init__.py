"""fp64 CPU oracle of the Gated DeltaNet-2 mixer -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never loads it and the
two share no code.  The arithmetic lives in ``gdn2_oracle.c`` (plain C, fp64,
token by token, OpenMP over independent heads); this module only compiles it
and marshals numpy arrays.

Source of the method: "Why NVIDIA Gated DeltaNet-2 separates erase and write
gates" (axbrief), section "Gated Delta Rule-2: per-channel erase/write split"
(recurrence and gate definitions; the gate-aware backward is the reverse-time
adjoint of that recurrence).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn2_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile gdn2_oracle.c into liboracle.so (gcc, -O2, OpenMP), and the
    layer oracle (gdn2_layer_oracle.c) beside it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    _load_layer()
    return _LIB


class _Lib:
    """ctypes binding of one compiled oracle library (the default build, or a
    deliberately mutated copy that a test compiles to check a pin fails)."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.oracle_fwd.argtypes = [P] * 9 + [I] * 5
        lib.oracle_fwd.restype = None
        lib.oracle_decode.argtypes = [P] * 8 + [I] * 4
        lib.oracle_decode.restype = None
        lib.oracle_bwd.argtypes = [P] * 16 + [I] * 5
        lib.oracle_bwd.restype = None
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = I
        self.lib = lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = _Lib(_LIB).lib
    return _lib


def compile_variant(src_text: str, out_path: str) -> "OracleFunctions":
    """Compile an edited copy of the oracle source (used by tests that plant a
    mistake and check that a pin catches it) and return its bound functions."""
    src = out_path + ".c"
    with open(src, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                           "-o", out_path, src, "-lm"])
    return OracleFunctions(_Lib(out_path).lib)


def source_text() -> str:
    with open(_SRC) as f:
        return f.read()


def _f64(x):
    return None if x is None else np.ascontiguousarray(x, dtype=np.float64)


def _ptr(x):
    return None if x is None else x.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return _load().oracle_num_threads()


class OracleFunctions:
    """fwd / decode / bwd bound to one compiled oracle library."""

    def __init__(self, lib):
        self.lib = lib

    def fwd(self, q, k, v, log_alpha, b, w, S0=None):
        """Token-by-token forward.  Token tensors [B,T,H,D]; S0 [B,H,dk,dv] or None.

        Returns (o [B,T,H,dv], S_T [B,H,dk,dv]) as float64.
        """
        q, k, v, la, bg, wg, S0 = map(_f64, (q, k, v, log_alpha, b, w, S0))
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        assert k.shape == la.shape == bg.shape == q.shape
        assert v.shape == wg.shape == (B, T, H, dv)
        if S0 is not None:
            assert S0.shape == (B, H, dk, dv)
        o = np.zeros((B, T, H, dv))
        ST = np.zeros((B, H, dk, dv))
        self.lib.oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(bg), _ptr(wg), _ptr(S0),
                           _ptr(o), _ptr(ST), B, T, H, dk, dv)
        return o, ST

    def decode(self, q, k, v, log_alpha, b, w, S):
        """One token per head: tokens [B,H,D], state [B,H,dk,dv].

        Returns (o [B,H,dv], S_new) without modifying the caller's S.
        """
        q, k, v, la, bg, wg = map(_f64, (q, k, v, log_alpha, b, w))
        S = np.array(S, dtype=np.float64, order="C", copy=True)
        B, H, dk = q.shape
        dv = v.shape[-1]
        assert S.shape == (B, H, dk, dv)
        o = np.zeros((B, H, dv))
        self.lib.oracle_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(bg), _ptr(wg), _ptr(S),
                              _ptr(o), B, H, dk, dv)
        return o, S

    def bwd(self, q, k, v, log_alpha, b, w, S0, dO, dS_T=None):
        """Reverse-time gate-aware VJP of L = sum <dO, o> + <dS_T, S_T>.

        Returns dict with dq, dk, dv, dlog_alpha, db, dw, dS0 (float64).
        """
        q, k, v, la, bg, wg, S0, dO, dST = map(_f64, (q, k, v, log_alpha, b, w, S0, dO, dS_T))
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        assert dO.shape == v.shape
        out = {n: np.zeros(q.shape) for n in ("dq", "dk", "dlog_alpha", "db")}
        out.update({n: np.zeros(v.shape) for n in ("dv", "dw")})
        out["dS0"] = np.zeros((B, H, dk, dv))
        self.lib.oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(bg), _ptr(wg), _ptr(S0),
                           _ptr(dO), _ptr(dST), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                           _ptr(out["dlog_alpha"]), _ptr(out["db"]), _ptr(out["dw"]), _ptr(out["dS0"]),
                           B, T, H, dk, dv)
        return out


def _default() -> OracleFunctions:
    return OracleFunctions(_load())


def fwd(*a, **kw):
    return _default().fwd(*a, **kw)


def decode(*a, **kw):
    return _default().decode(*a, **kw)


def bwd(*a, **kw):
    return _default().bwd(*a, **kw)


# ---------------------------------------------------------------------------
# The layer prologue and epilogue (gdn2_layer_oracle.c): short causal
# convolution + SiLU (+ L2 norm) of the q/k/v paths, the gate activations and
# the RMS-normalised, SiLU-gated output, with their backward passes.

_LAYER_SRC = os.path.join(_HERE, "gdn2_layer_oracle.c")
_LAYER_LIB = os.path.join(_HERE, "liblayer_oracle.so")
_layer = None


def _load_layer():
    global _layer
    if _layer is None:
        if not os.path.exists(_LAYER_LIB) or os.path.getmtime(_LAYER_LIB) < os.path.getmtime(_LAYER_SRC):
            tmp = _LAYER_LIB + ".tmp%d" % os.getpid()
            subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c99", "-o", tmp, _LAYER_SRC, "-lm"])
            os.replace(tmp, _LAYER_LIB)
        lib = ctypes.CDLL(_LAYER_LIB)
        P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        lib.oracle_prologue_path.argtypes = [P, P, I, P, I, I, I, I, I, P, P]
        lib.oracle_prologue_path_bwd.argtypes = [P, P, I, P, P, P, I, I, I, I, I, P, P, P]
        lib.oracle_gate.argtypes = [P, P, Z, I]
        lib.oracle_gate_bwd.argtypes = [P, P, P, Z, I]
        lib.oracle_epilogue.argtypes = [P, P, P, P, I, I, I, I]
        lib.oracle_epilogue_bwd.argtypes = [P, P, P, P, P, P, P, I, I, I, I]
        for f in ("oracle_prologue_path", "oracle_prologue_path_bwd", "oracle_gate", "oracle_gate_bwd",
                  "oracle_epilogue", "oracle_epilogue_bwd"):
            getattr(lib, f).restype = None
        _layer = lib
    return _layer


def prologue_path(x, W, l2):
    """One input path: depthwise causal conv (W [H*D][K]) + SiLU, and for the
    query/key paths (l2=True) the L2 norm over the head dim.  x [B,T,H,D]."""
    x, W = _f64(x), _f64(W)
    B, T, H, D = x.shape
    K = W.shape[-1]
    assert W.shape == (H * D, K)
    out, yw, sw = np.zeros(x.shape), np.zeros(x.shape), np.zeros(x.shape)
    _load_layer().oracle_prologue_path(_ptr(x), _ptr(W), K, _ptr(out), B, T, H, D, int(bool(l2)), _ptr(yw), _ptr(sw))
    return out


def prologue_path_bwd(x, W, dout, l2):
    """Backward of prologue_path: (dx [B,T,H,D], dW [H*D][K])."""
    x, W, dout = _f64(x), _f64(W), _f64(dout)
    B, T, H, D = x.shape
    K = W.shape[-1]
    dx, dW = np.zeros(x.shape), np.zeros(W.shape)
    work = [np.zeros(x.shape) for _ in range(3)]
    _load_layer().oracle_prologue_path_bwd(_ptr(x), _ptr(W), K, _ptr(dout), _ptr(dx), _ptr(dW), B, T, H, D,
                                           int(bool(l2)), *[_ptr(w) for w in work])
    return dx, dW


def gate(x, kind):
    """kind 'log_alpha': log sigmoid(x); 'sigmoid': sigmoid(x)."""
    x = _f64(x)
    out = np.zeros(x.shape)
    _load_layer().oracle_gate(_ptr(x), _ptr(out), x.size, 0 if kind == "log_alpha" else 1)
    return out


def gate_bwd(x, dout, kind):
    x, dout = _f64(x), _f64(dout)
    dx = np.zeros(x.shape)
    _load_layer().oracle_gate_bwd(_ptr(x), _ptr(dout), _ptr(dx), x.size, 0 if kind == "log_alpha" else 1)
    return dx


def epilogue(o, g, gamma):
    """z = o / rms(o) * gamma * silu(g) per token and head; o, g [B,T,H,D], gamma [D]."""
    o, g, gamma = _f64(o), _f64(g), _f64(gamma)
    B, T, H, D = o.shape
    z = np.zeros(o.shape)
    _load_layer().oracle_epilogue(_ptr(o), _ptr(g), _ptr(gamma), _ptr(z), B, T, H, D)
    return z


def epilogue_bwd(o, g, gamma, dz):
    """Backward of epilogue: (do, dg, dgamma)."""
    o, g, gamma, dz = _f64(o), _f64(g), _f64(gamma), _f64(dz)
    B, T, H, D = o.shape
    dO, dg, dgamma = np.zeros(o.shape), np.zeros(o.shape), np.zeros(D)
    _load_layer().oracle_epilogue_bwd(_ptr(o), _ptr(g), _ptr(gamma), _ptr(dz), _ptr(dO), _ptr(dg), _ptr(dgamma),
                                      B, T, H, D)
    return dO, dg, dgamma
