"""Helpers of the GPU parity tests: device copies of seeded inputs and the
error measures of the tolerance (relative L2 over the whole tensor, max-abs)."""
import os

import numpy as np

NAMES = ("q", "k", "v", "log_alpha", "b", "w")
# bf16 tokens with an fp32 state: rel-L2 <= 1e-2 and max-abs <= 5e-2 on o,
# S_T and every gradient; fp32 tokens: rel-L2 <= 1e-4.
TOL_BF16 = dict(rel=1e-2, abs=5e-2)
# Outputs whose entries grow well past one (the gated output z, whose entries
# reach ~10, and the gradients of the reduced-gate forms, where uniform gates
# push |dk| to ~15): a bf16 value of magnitude x is itself rounded by up to
# 2^-8 x, so each entry is held to 5e-2 + 2^-7 |ref| (the stated bound plus
# the relative rounding of one bf16 result and of the fp32 path before it),
# with the same rel-L2 <= 1e-2 over the tensor.
TOL_BF16_ELEM = dict(rel=1e-2, abs=5e-2, abs_rel=2.0 ** -7)


def check_sum(name, x, ref, ref_abs):
    """A gradient that is a sum of per-channel terms (dbeta = sum_c db + sum_j
    dw; a scalar decay's gradient = sum_c dlog_alpha): the terms' errors add,
    so each entry is held to 5e-2 + 2^-7 * (the sum of the terms' magnitudes,
    ref_abs) -- the usual bound of a summation -- with rel-L2 <= 1e-2."""
    r = rel_l2(x, ref)
    assert np.all(np.isfinite(x)), "%s: non-finite values" % name
    err = np.abs(np.asarray(x, np.float64) - np.asarray(ref, np.float64))
    worst = float(np.max(err - (5e-2 + 2.0 ** -7 * np.asarray(ref_abs, np.float64))))
    if os.environ.get("GDN2_REPORT"):
        print("parity %-28s rel-L2 %.3e (<= 1e-02)  max(err - bound) %.4f (<= 0)" % (name, r, worst))
    assert r <= 1e-2 and worst <= 0, "%s: rel-L2 %.3e, an entry exceeds its sum bound by %.3e" % (name, r, worst)
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
    if "abs_rel" in tol and np.size(ref):  # per element: abs + abs_rel |ref|
        err = np.abs(np.asarray(x, np.float64) - np.asarray(ref, np.float64))
        lim = tol["abs"] + tol["abs_rel"] * np.abs(np.asarray(ref, np.float64))
        worst = float(np.max(err - lim))
        if os.environ.get("GDN2_REPORT"):
            print("parity %-28s rel-L2 %.3e (<= %.0e)  max(err - bound) %.4f (<= 0)" % (name, r, tol["rel"], worst))
        assert r <= tol["rel"] and worst <= 0, "%s: rel-L2 %.3e, an entry exceeds 5e-2 + 2^-7|ref| by %.3e" % (
            name, r, worst)
        return r, m
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
