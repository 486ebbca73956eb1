"""A bounded device wait that runs out: with a short wait limit, the forward
withholds the arrival that hands one chunk's intra-chunk results to its
state chain, so the chain's wait for it ends without it.  The kernel must
give up cleanly -- no copy or tensor-core operation in flight, tensor memory
freed -- and record GDN2_ERR_TIMEOUT in the device status word; the next
normal call on the same context must be clean and match the oracle.  (No
fault, trap or endless wait is involved: the wait is bounded.)"""
import numpy as np
import pytest

import oracle
from gpu_util import NAMES, TOL_BF16, check, dev_state, host, tokens
from gated_delta_rule_gdn2_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu


def test_withheld_arrival_times_out_and_context_stays_usable():
    import torch
    import gated_delta_rule_gdn2_b200 as g
    x = make_inputs(1, 320, 2, 128, 128, seed=5, dtype="bf16")
    toks = tokens(x, "bf16")
    S0 = dev_state(x["S0"])
    assert g.gdn2_get_device_status() == 0
    try:
        assert g.gdn2_debug_set(g.GDN2_DEBUG_WAIT_LIMIT, 1 << 12) == 0
        assert g.gdn2_debug_set(g.GDN2_DEBUG_WITHHOLD_READY, 2) == 0
        o = torch.empty((1, 320, 2, 128), dtype=torch.bfloat16, device="cuda")
        ST = torch.empty((1, 2, 128, 128), dtype=torch.float32, device="cuda")
        ws = torch.empty(2 * 64 * 128 * 4, dtype=torch.uint8, device="cuda")
        st = g.gdn2_chunk_fwd(*toks, S0, o, ST, 1, 320, 2, 128, 128, g.GDN2_BF16, ws, ws.numel())
        assert st == 0  # the launch itself is fine
        assert g.gdn2_get_device_status() == -4  # GDN2_ERR_TIMEOUT, read and cleared
        assert g.gdn2_get_device_status() == 0
    finally:
        g.gdn2_debug_set(g.GDN2_DEBUG_WITHHOLD_READY, -1)
        g.gdn2_debug_set(g.GDN2_DEBUG_WAIT_LIMIT, 0)
    o, ST = g.chunk_fwd(*toks, S0=S0)
    assert g.gdn2_get_device_status() == 0
    o_ref, ST_ref = oracle.fwd(*[x[n] for n in NAMES], x["S0"])
    check("o", host(o), o_ref, TOL_BF16)
    check("S_T", host(ST), ST_ref, TOL_BF16)


def test_debug_knobs_reject_bad_values():
    import gated_delta_rule_gdn2_b200 as g
    assert g.gdn2_debug_set(7, 0) == -1
    assert g.gdn2_debug_set(g.GDN2_DEBUG_WAIT_LIMIT, -1) == -1
    assert g.gdn2_debug_set(g.GDN2_DEBUG_WITHHOLD_READY, -2) == -1
    assert g.gdn2_debug_set(g.GDN2_DEBUG_WITHHOLD_READY, -1) == 0
