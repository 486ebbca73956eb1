"""Packed variable-length batches (gdn2_chunk_fwd_varlen / _bwd_varlen and the
saved-state pair) against the fp64 oracle run on each sequence alone, through
the C ABI: ragged lengths below, at and above the 64-token chunk, lengths
that are not a multiple of 64, and an empty sequence.  A packed batch of
equal lengths must give the fixed-length call's results bit for bit."""
import numpy as np
import pytest

import oracle
from gpu_util import NAMES, TOL_BF16, TOL_FP32, check, dev, dev_state, host
from gated_delta_rule_gdn2_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu
GRADS = ("dq", "dk", "dv", "dlog_alpha", "db", "dw")


def packed(lens, H, dk, dv, dtype, seed):
    """Token tensors [total, H, D] of len(lens) sequences, S0 [N, H, dk, dv],
    dO, a nonzero dS_T and the offsets."""
    total = int(sum(lens))
    x = make_inputs(1, max(total, 1), H, dk, dv, seed=seed, dtype=dtype, with_do=True)
    out = {n: x[n][0, :total] for n in NAMES + ("dO",)}
    rng = np.random.default_rng(seed)
    out["S0"] = (0.02 * rng.standard_normal((len(lens), H, dk, dv))).astype(np.float32)
    out["dST"] = (0.1 * rng.standard_normal((len(lens), H, dk, dv))).astype(np.float32)
    out["cu"] = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return out


def oracle_per_sequence(x, lens, H, dk, dv):
    o = np.zeros(x["v"].shape)
    ST = np.zeros((len(lens), H, dk, dv))
    g = {n: np.zeros(x["q" if n in ("dq", "dk", "dlog_alpha", "db") else "v"].shape) for n in GRADS}
    dS0 = np.zeros((len(lens), H, dk, dv))
    for n, (r0, r1) in enumerate(zip(x["cu"][:-1], x["cu"][1:])):
        if r1 == r0:  # an empty sequence passes its state through
            ST[n] = x["S0"][n]
            dS0[n] = x["dST"][n]
            continue
        seq = {m: x[m][None, r0:r1] for m in NAMES + ("dO",)}
        o_n, S_n = oracle.fwd(*[seq[m] for m in NAMES], x["S0"][n:n + 1])
        o[r0:r1] = o_n[0]
        ST[n] = S_n[0]
        gr = oracle.bwd(*[seq[m] for m in NAMES], x["S0"][n:n + 1], seq["dO"], x["dST"][n:n + 1])
        for m in GRADS:
            g[m][r0:r1] = gr[m][0]
        dS0[n] = gr["dS0"][0]
    return o, ST, g, dS0


CASES = [
    ((0, 1, 63, 64, 65, 200, 130), 128, 128),
    ((70, 0, 129, 5), 64, 128),
    ((33, 128, 1), 128, 64),
]


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("lens,dk,dv", CASES)
def test_varlen_matches_per_sequence_oracle(lens, dk, dv, dtype):
    import torch
    import gated_delta_rule_gdn2_b200 as g
    H = 2
    x = packed(lens, H, dk, dv, dtype, seed=500 + sum(lens) + dk)
    toks = [dev(x[n], dtype) for n in NAMES]
    cu = torch.from_numpy(x["cu"]).cuda()
    S0 = dev_state(x["S0"])
    o, ST = g.chunk_fwd_varlen(*toks, cu, S0=S0)
    gr = g.chunk_bwd_varlen(*toks, cu, S0, dev(x["dO"], dtype), dev_state(x["dST"]))
    assert g.gdn2_get_device_status() == 0
    o_ref, ST_ref, g_ref, dS0_ref = oracle_per_sequence(x, lens, H, dk, dv)
    tol = TOL_BF16 if dtype == "bf16" else TOL_FP32
    check("o", host(o), o_ref, tol)
    check("S_T", host(ST), ST_ref, tol)
    for n in GRADS:
        check(n, host(gr[n]), g_ref[n], tol)
    check("dS0", host(gr["dS0"]), dS0_ref, tol)
    if dtype == "bf16":
        # the saved-state pair: the same results bit for bit
        o2, ST2, states = g.chunk_fwd_varlen(*toks, cu, S0=S0, save_states=True)
        gr2 = g.chunk_bwd_varlen(*toks, cu, S0, dev(x["dO"], dtype), dev_state(x["dST"]), states=states)
        assert g.gdn2_get_device_status() == 0
        np.testing.assert_array_equal(host(o2), host(o))
        np.testing.assert_array_equal(host(ST2), host(ST))
        for n in GRADS + ("dS0",):
            np.testing.assert_array_equal(host(gr2[n]), host(gr[n]))


@pytest.mark.parametrize("T", [150, 256])
def test_equal_lengths_match_fixed_length_call(T):
    """N sequences of T tokens packed give exactly the [N, T, H, D] results."""
    import torch
    import gated_delta_rule_gdn2_b200 as g
    N, H, d = 3, 2, 128
    x = make_inputs(N, T, H, d, d, seed=77 + T, dtype="bf16", with_do=True)
    toks = [dev(x[n], "bf16") for n in NAMES]
    S0 = dev_state(x["S0"])
    dO = dev(x["dO"], "bf16")
    o1, S1 = g.chunk_fwd(*toks, S0=S0)
    g1 = g.chunk_bwd(*toks, S0, dO)
    cu = torch.arange(0, (N + 1) * T, T, dtype=torch.int32, device="cuda")
    flat = [t.reshape(N * T, H, d) for t in toks]
    o2, S2 = g.chunk_fwd_varlen(*flat, cu, S0=S0)
    g2 = g.chunk_bwd_varlen(*flat, cu, S0, dO.reshape(N * T, H, d))
    assert g.gdn2_get_device_status() == 0
    np.testing.assert_array_equal(host(o2).reshape(host(o1).shape), host(o1))
    np.testing.assert_array_equal(host(S2), host(S1))
    for n in GRADS:
        np.testing.assert_array_equal(host(g2[n]).reshape(host(g1[n]).shape), host(g1[n]))
    np.testing.assert_array_equal(host(g2["dS0"]), host(g1["dS0"]))


def test_out_of_range_offsets_are_reported():
    """Offsets that decrease are caught on the device: that sequence is left
    alone, the others run, and the status word says GDN2_ERR_INVALID_ARG."""
    import torch
    import gated_delta_rule_gdn2_b200 as g
    lens_ok = (100, 50)
    x = packed(lens_ok, 1, 128, 128, "bf16", seed=9)
    toks = [dev(x[n], "bf16") for n in NAMES]
    cu = torch.tensor([0, 100, 20, 150], dtype=torch.int32, device="cuda")  # sequence 1: 100 -> 20
    S0 = torch.zeros((3, 1, 128, 128), device="cuda")
    o = torch.zeros((150, 1, 128), dtype=torch.bfloat16, device="cuda")
    ST = torch.full((3, 1, 128, 128), 7.0, device="cuda")
    nws = g.gdn2_chunk_fwd_varlen_workspace(3, 150, 1, 128, 128, g.GDN2_BF16)
    ws = torch.empty(nws, dtype=torch.uint8, device="cuda")
    st = g.gdn2_chunk_fwd_varlen(*toks, S0, o, ST, cu, 3, 150, 1, 128, 128, g.GDN2_BF16, ws, nws)
    assert st == 0
    assert g.gdn2_get_device_status() == -1
    assert g.gdn2_get_device_status() == 0  # read and cleared
    assert float(ST[1].min()) == 7.0 and float(ST[1].max()) == 7.0  # untouched
