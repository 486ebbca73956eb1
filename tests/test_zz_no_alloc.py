"""gdn2_chunk_fwd_noalloc: the forward for callers that cannot allocate device
memory (no cudaMalloc available to them, or a path that must not allocate).
Through the C ABI, its outputs must equal those of gdn2_chunk_fwd with a
caller-provided workspace, on two calls in a row that share the library's
fixed scratch array.  The first input set has chunks decaying past e^-64, so
the forward's scratch is really used.  (File named to be collected last.)"""
import numpy as np
import pytest

from gpu_util import TOL_BF16, check, dev_state, host, tokens
from gated_delta_rule_gdn2_b200.inputs import make_inputs, round_bf16

pytestmark = pytest.mark.gpu


def _inputs(fast_decay, seed):
    x = make_inputs(2, 200, 3, 128, 128, seed=seed, dtype="bf16")
    if fast_decay:
        rng = np.random.default_rng(seed)
        la = x["log_alpha"]
        m = rng.random(la.shape) < 0.05
        la[m] = -40.0 * rng.random(m.sum()).astype(np.float32)
        x["log_alpha"] = round_bf16(la)
    return x


def _noalloc(x):
    import torch
    import gated_delta_rule_gdn2_b200 as g
    q, k, v, la, b, w = tokens(x, "bf16")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device="cuda")
    ST = torch.empty((B, H, dk, dv), dtype=torch.float32, device="cuda")
    st = g.gdn2_chunk_fwd_noalloc(q, k, v, la, b, w, dev_state(x["S0"]), o, ST, B, T, H, dk, dv,
                                  g.GDN2_BF16)
    assert st == 0, g.gdn2_status_string(st)
    assert g.gdn2_get_device_status() == 0
    return host(o), host(ST)


def test_noalloc_matches_chunk_fwd_two_calls():
    import gated_delta_rule_gdn2_b200 as g
    for fast_decay, seed in ((True, 31), (False, 32)):
        x = _inputs(fast_decay, seed)
        o_na, S_na = _noalloc(x)
        o_ref, S_ref = g.chunk_fwd(*tokens(x, "bf16"), S0=dev_state(x["S0"]))
        check("o", o_na, host(o_ref), TOL_BF16)
        check("S_T", S_na, host(S_ref), TOL_BF16)


def test_noalloc_rejects_oversized_problem():
    import gated_delta_rule_gdn2_b200 as g
    # B*H*dk = 257*128 > 32768: refused before any launch (pointers unused)
    st = g.gdn2_chunk_fwd_noalloc(256, 256, 256, 256, 256, 256, None, 256, None, 257, 64, 1, 128, 128,
                                  g.GDN2_BF16)
    assert st == -5
