"""Helpers of the GPU parity tests: device copies of seeded inputs and the
error measures of the tolerance (relative L2 over the whole tensor, max-abs)."""
import os

import numpy as np

NAMES = ("q", "k", "v", "log_alpha", "b", "w")
# bf16 tokens with an fp32 state: rel-L2 <= 1e-2 and max-abs <= 5e-2 on o,
# S_T and every gradient; fp32 tokens: rel-L2 <= 1e-4.
TOL_BF16 = dict(rel=1e-2, abs=5e-2)
TOL_FP32 = dict(rel=1e-4, abs=1e-3)


def rel_l2(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (den if den > 0 else 1.0))


def max_abs(x, ref):
    return float(np.max(np.abs(np.asarray(x, np.float64) - np.asarray(ref, np.float64)))) if np.size(ref) else 0.0


def check(name, x, ref, tol):
    r, m = rel_l2(x, ref), max_abs(x, ref)
    assert np.all(np.isfinite(x)), "%s: non-finite values" % name
    bound = tol["abs"]
    if os.environ.get("GDN2_REPORT"):
        print("parity %-28s rel-L2 %.3e (<= %.0e)  max-abs %.4f (<= %.3g)" % (name, r, tol["rel"], m, bound))
    assert r <= tol["rel"] and m <= bound, "%s: rel-L2 %.3e max-abs %.3e (bound %.3e, tol %s)" % (
        name, r, m, bound, tol)
    return r, m


def dev(x, dtype):
    import torch
    if x is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(device="cuda", dtype=torch.bfloat16 if dtype == "bf16" else torch.float32)


def dev_state(x):
    import torch
    return None if x is None else torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def host(t):
    return t.float().cpu().numpy().astype(np.float64)


def tokens(x, dtype):
    return [dev(x[n], dtype) for n in NAMES]


def sub_heads(x, heads):
    """Restrict token tensors [B,T,H,D] (and S0 [B,H,..]) to a list of (b, h)."""
    out = {}
    for n, v in x.items():
        if v is None:
            out[n] = None
        elif n == "S0":
            out[n] = np.stack([v[b, h] for b, h in heads])[:, None]
        else:
            out[n] = np.stack([v[b, :, h] for b, h in heads])[:, :, None]
    return out
