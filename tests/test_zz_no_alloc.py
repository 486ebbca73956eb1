"""gdn2_chunk_fwd_noalloc: the forward for callers that cannot allocate device
memory (no cudaMalloc available to them, or a path that must not allocate).
Through the C ABI, its outputs must equal those of gdn2_chunk_fwd given the
workspace gdn2_chunk_fwd_workspace asks for -- bit for bit, since the same
kernels run on the same inputs -- on two calls in a row that share the
library's fixed scratch array, and match the fp64 oracle.  The first input set
has chunks decaying past e^-64, so the forward's scratch is really used; the
B1 H1 T4096 case fits the sequence-segmented forward's workspace into the
fixed array, so it runs that path.  (File named to be collected last.)"""
import numpy as np
import pytest

import oracle
from gpu_util import NAMES, TOL_BF16, check, dev_state, host, tokens
from gated_delta_rule_gdn2_b200.inputs import make_inputs, round_bf16

pytestmark = pytest.mark.gpu


def _inputs(fast_decay, seed, B=2, T=200, H=3):
    x = make_inputs(B, T, H, 128, 128, seed=seed, dtype="bf16")
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


@pytest.mark.parametrize("case", ["plain", "segmented"])
def test_noalloc_matches_chunk_fwd_two_calls(case):
    import gated_delta_rule_gdn2_b200 as g
    if case == "plain":
        sets = [_inputs(True, 31), _inputs(False, 32)]
    else:
        # one long sequence: the segmented forward, whose workspace fits the array
        B, T, H = 1, 4096, 1
        assert g.gdn2_chunk_fwd_workspace(B, T, H, 128, 128, g.GDN2_BF16) > B * H * 64 * 128 * 4
        sets = [_inputs(False, 33, B, T, H), _inputs(False, 34, B, T, H)]
    for x in sets:
        o_na, S_na = _noalloc(x)
        o_ref, S_ref = g.chunk_fwd(*tokens(x, "bf16"), S0=dev_state(x["S0"]))
        np.testing.assert_array_equal(o_na, host(o_ref))
        np.testing.assert_array_equal(S_na, host(S_ref))
        o_or, S_or = oracle.fwd(*[x[n] for n in NAMES], x["S0"])
        check("o", o_na, o_or, TOL_BF16)
        check("S_T", S_na, S_or, TOL_BF16)


def test_noalloc_rejects_oversized_problem():
    import gated_delta_rule_gdn2_b200 as g
    # B*H*dk = 257*128 > 32768: refused before any launch (pointers unused)
    st = g.gdn2_chunk_fwd_noalloc(256, 256, 256, 256, 256, 256, None, 256, None, 257, 64, 1, 128, 128,
                                  g.GDN2_BF16)
    assert st == -5
