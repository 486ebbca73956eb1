"""Seeded synthetic inputs for the Gated DeltaNet-2 mixer.

This module holds the input recipe only -- none of the mixer's arithmetic --
so that the CUDA path and the CPU oracle can be fed identical values.

Recipe (shapes and distributions of the 1.3B-layer workloads; the pages train
on FineWeb-Edu text at 4K context, which is not available here, so seeded
normals stand in for the projected activations):

* q, k ~ N(0, 1), then L2-normalised over the head dimension per (b, t, h)
  (the q/k path ends in an L2 norm: "Why NVIDIA Gated DeltaNet-2 separates
  erase and write gates", section on implications for practitioners).
* v ~ N(0, 1).
* alpha = sigmoid(x), x ~ N(mu_alpha, 1) per key channel, passed on as
  log_alpha = -softplus(-x) (mu_alpha = 3, or 4 for the slow-decay long runs).
* b = sigmoid(N(0,1)) per key channel, w = sigmoid(N(0,1)) per value channel.
* S0 = s0_std * N(0, 1) in fp32 (0.02, or an all-zero state).
* do ~ N(0, 1) for the backward workloads.

Draws come from ``numpy.random.Generator(PCG64(seed))`` in the fixed order
q, k, v, x_alpha, x_b, x_w, S0, do, each drawn in float32.  For bf16 workloads
every token tensor (and do) is then rounded to bfloat16 with
round-to-nearest-even; the fp32 values of those bf16 numbers are what both the
GPU and the oracle consume.  Decode step s draws from PCG64([seed, s]).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

TOKEN_NAMES = ("q", "k", "v", "log_alpha", "b", "w")


@dataclass
class Workload:
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    dtype: str  # "bf16" or "fp32": dtype of every token tensor
    seed: int
    alpha_mu: float = 3.0
    s0_std: float = 0.02
    with_do: bool = False
    extra: dict = field(default_factory=dict)


# The five workloads of the pages' shapes (tiny parity case, 1.3B-layer
# prefill, batched decode, long-sequence forward, training fwd+bwd).
WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 1, 256, 2, 64, 64, "fp32", 1000, s0_std=0.0),
    "prefill": Workload("prefill", 8, 4096, 16, 128, 128, "bf16", 1001),
    "decode": Workload("decode", 256, 1, 16, 128, 128, "bf16", 1002, extra={"steps": 1024}),
    "long": Workload("long", 1, 8192, 16, 128, 128, "bf16", 1003, alpha_mu=4.0,
                     extra={"T_list": (8192, 32768, 131072)}),
    "train": Workload("train", 8, 4096, 16, 128, 128, "bf16", 1004, with_do=True),
}


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even), kept as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if x.ndim > 0 and x.size > (1 << 22):
        return _blockwise(_round_bf16, x)
    return _round_bf16(x)


def _round_bf16(x):
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    nan = np.isnan(x)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16) << 16
    out = r.astype(np.uint32).view(np.float32)
    if nan.any():
        out = out.copy()
        out[nan] = np.nan
    return out


def _blockwise(f, x, rows=1 << 14):
    """f applied to blocks of rows of x (last axis kept whole): the same
    values as f(x), with temporaries that stay in cache on long inputs."""
    x = np.ascontiguousarray(x)
    if x.ndim == 0 or x.size <= rows * x.shape[-1]:
        return f(x)
    flat = x.reshape(-1, x.shape[-1])
    out = np.empty(flat.shape, dtype=np.float32)
    for i in range(0, flat.shape[0], rows):
        out[i:i + rows] = f(flat[i:i + rows])
    return out.reshape(x.shape)


def _sigmoid(x):
    return _blockwise(lambda y: (1.0 / (1.0 + np.exp(-y.astype(np.float64)))).astype(np.float32), x)


def _log_sigmoid(x):
    return _blockwise(lambda y: (-np.logaddexp(0.0, -y.astype(np.float64))).astype(np.float32), x)


def _unit_rows(x):
    n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    return (x / np.maximum(n, 1e-30)).astype(np.float32)


def _unit(x):
    return _blockwise(_unit_rows, x)


def draw_tokens(rng: np.random.Generator, lead: tuple, dk: int, dv: int, alpha_mu: float,
                dtype: str) -> dict:
    """q, k, v, log_alpha, b, w with leading shape ``lead`` (e.g. (B,T,H) or (B,H))."""
    q = _unit(rng.standard_normal(lead + (dk,), dtype=np.float32))
    k = _unit(rng.standard_normal(lead + (dk,), dtype=np.float32))
    v = rng.standard_normal(lead + (dv,), dtype=np.float32)
    xa = rng.standard_normal(lead + (dk,), dtype=np.float32) + np.float32(alpha_mu)
    xb = rng.standard_normal(lead + (dk,), dtype=np.float32)
    xw = rng.standard_normal(lead + (dv,), dtype=np.float32)
    out = {"q": q, "k": k, "v": v, "log_alpha": _log_sigmoid(xa), "b": _sigmoid(xb),
           "w": _sigmoid(xw)}
    if dtype == "bf16":
        out = {n: round_bf16(x) for n, x in out.items()}
    return out


def make_inputs(B: int, T: int, H: int, dk: int, dv: int, *, seed: int, dtype: str = "bf16",
                alpha_mu: float = 3.0, s0_std: float = 0.02, with_do: bool = False) -> dict:
    """Token tensors [B,T,H,D] (float32 holding bf16 values when dtype='bf16'),
    S0 [B,H,dk,dv] float32 (None when s0_std == 0), and dO when requested."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out = draw_tokens(rng, (B, T, H), dk, dv, alpha_mu, dtype)
    if s0_std > 0:
        out["S0"] = (np.float32(s0_std) * rng.standard_normal((B, H, dk, dv), dtype=np.float32))
    else:
        out["S0"] = None
    if with_do:
        do = rng.standard_normal((B, T, H, dv), dtype=np.float32)
        out["dO"] = round_bf16(do) if dtype == "bf16" else do
    return out


def make_workload(w: Workload, T: int | None = None) -> dict:
    return make_inputs(w.B, T if T is not None else w.T, w.H, w.dk, w.dv, seed=w.seed,
                       dtype=w.dtype, alpha_mu=w.alpha_mu, s0_std=w.s0_std, with_do=w.with_do)


def decode_step_inputs(B: int, H: int, dk: int, dv: int, *, seed: int, step: int,
                       dtype: str = "bf16", alpha_mu: float = 3.0) -> dict:
    """Tokens [B,H,D] for decode step ``step`` drawn from PCG64([seed, step])."""
    rng = np.random.Generator(np.random.PCG64([seed, step]))
    return draw_tokens(rng, (B, H), dk, dv, alpha_mu, dtype)


def decode_initial_state(B: int, H: int, dk: int, dv: int, *, seed: int,
                         s0_std: float = 0.02) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64([seed, 1 << 30]))
    return np.float32(s0_std) * rng.standard_normal((B, H, dk, dv), dtype=np.float32)


def make_inputs_device(B: int, T: int, H: int, dk: int, dv: int, *, seed: int, device,
                       alpha_mu: float = 3.0, s0_std: float = 0.02):
    """The same distributions as make_inputs, drawn on the GPU with torch's
    seeded generator (for benchmark inputs of hundreds of millions of values,
    which the host generator takes minutes to draw).  Token tensors bf16
    [B,T,H,D], S0 fp32 [B,H,dk,dv].  Not the values make_inputs gives: the
    parity tests use make_inputs."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    lead = (B, T, H)

    def n(*shape):
        return torch.randn(shape, generator=g, device=device, dtype=torch.float32)

    q = torch.nn.functional.normalize(n(*lead, dk), dim=-1)
    k = torch.nn.functional.normalize(n(*lead, dk), dim=-1)
    v = n(*lead, dv)
    la = torch.nn.functional.logsigmoid(n(*lead, dk) + alpha_mu)
    b = torch.sigmoid(n(*lead, dk))
    w = torch.sigmoid(n(*lead, dv))
    out = {name: t.to(torch.bfloat16) for name, t in zip(TOKEN_NAMES, (q, k, v, la, b, w))}
    out["S0"] = s0_std * n(B, H, dk, dv)
    return out
