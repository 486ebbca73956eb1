"""GPU parity of gdn2_decode_step against the oracle through the C ABI, and
against the chunk forward (T decode steps = one chunk-forward call)."""
import numpy as np
import pytest

import oracle
from gpu_util import TOL_BF16, TOL_FP32, NAMES, check, dev, dev_state, host, tokens
from gated_delta_rule_gdn2_b200.inputs import (WORKLOADS, decode_initial_state, decode_step_inputs,
                                             make_inputs)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_decode_steps_match_oracle(dk, dv, dtype):
    import gated_delta_rule_gdn2_b200 as g
    B, H = 3, 5
    S = decode_initial_state(B, H, dk, dv, seed=7)
    Sd = dev_state(S)
    Sref = S.astype(np.float64)
    tol = TOL_BF16 if dtype == "bf16" else TOL_FP32
    for s in range(20):
        x = decode_step_inputs(B, H, dk, dv, seed=7, step=s, dtype=dtype)
        o = g.decode_step(*tokens(x, dtype), Sd)
        o_ref, Sref = oracle.decode(*[x[n] for n in NAMES], Sref)
        check("o step %d" % s, host(o), o_ref, tol)
    check("S", host(Sd), Sref, tol)
    assert g.gdn2_get_device_status() == 0


def test_decode_full_batch_1_16_1024_steps():
    """B=256, H=16, d=128 state resident and updated in place for 1024 steps;
    compared with the oracle after 1, 16 and 1024 steps on sampled heads."""
    import gated_delta_rule_gdn2_b200 as g
    w = WORKLOADS["decode"]
    B, H, d = w.B, w.H, w.dk
    S = decode_initial_state(B, H, d, d, seed=w.seed)
    Sd = dev_state(S)
    heads = [(0, 0), (100, 5), (255, 15)]
    Sref = np.stack([S[b, h] for b, h in heads])[:, None].astype(np.float64)
    for s in range(1024):
        x = decode_step_inputs(B, H, d, d, seed=w.seed, step=s)
        o = g.decode_step(*tokens(x, "bf16"), Sd)
        xs = {n: np.stack([x[n][b, h] for b, h in heads])[:, None] for n in NAMES}
        o_ref, Sref = oracle.decode(*[xs[n] for n in NAMES], Sref)
        if s + 1 in (1, 16, 1024):
            oh = host(o)
            Sh = host(Sd)
            for i, (b, h) in enumerate(heads):
                check("o step %d head %s" % (s + 1, (b, h)), oh[b, h], o_ref[i, 0], TOL_BF16)
                check("S step %d head %s" % (s + 1, (b, h)), Sh[b, h], Sref[i, 0], TOL_BF16)
            assert np.all(np.isfinite(Sh))


def test_decode_equals_chunk_forward():
    import torch
    import gated_delta_rule_gdn2_b200 as g
    x = make_inputs(2, 70, 3, 128, 128, seed=21, dtype="bf16")
    o_chunk, S_chunk = g.chunk_fwd(*tokens(x, "bf16"), S0=dev_state(x["S0"]))
    Sd = dev_state(x["S0"])
    outs = []
    for t in range(70):
        xt = [dev(np.ascontiguousarray(x[n][:, t]), "bf16") for n in NAMES]
        outs.append(host(g.decode_step(*xt, Sd)))
    o_dec = np.stack(outs, axis=1)
    check("o", o_dec, host(o_chunk), TOL_BF16)
    check("S", host(Sd), host(S_chunk), TOL_BF16)
    del torch
