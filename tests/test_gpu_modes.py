"""Reduced gates through the C ABI: KDA (one scalar beta per token and head
for both the erase and the write gate) and Gated DeltaNet (that, and a scalar
decay).  The forward must equal the general call with the gates expanded to
vectors bit for bit, and both passes must match the fp64 oracle run on the
expanded gates, whose reduction to these two models is pinned on the CPU
(test_oracle_pins.py); dbeta is checked against sum_c db + sum_j dw and a
scalar decay's gradient against sum_c dlog_alpha of the oracle."""
import numpy as np
import pytest

import oracle
from gpu_util import NAMES, TOL_BF16, TOL_BF16_ELEM, TOL_FP32, check, check_sum, dev, dev_state, host
from gated_delta_rule_gdn2_b200.inputs import make_inputs, round_bf16

pytestmark = pytest.mark.gpu


def reduced_inputs(B, T, H, dk, dv, mode, dtype, seed):
    """General inputs whose gates are scalars per (b, t, h), plus those scalars."""
    x = make_inputs(B, T, H, dk, dv, seed=seed, dtype=dtype, with_do=True)
    rng = np.random.default_rng(seed)
    beta = (1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))).astype(np.float32)
    la_s = (-np.logaddexp(0.0, -(rng.standard_normal((B, T, H)) + 3.0))).astype(np.float32)
    if dtype == "bf16":
        beta, la_s = round_bf16(beta), round_bf16(la_s)
    x["beta"] = beta
    x["b"] = np.repeat(beta[..., None], dk, axis=-1)
    x["w"] = np.repeat(beta[..., None], dv, axis=-1)
    if mode == "gdn":
        x["la_s"] = la_s
        x["log_alpha"] = np.repeat(la_s[..., None], dk, axis=-1)
    return x


def reduced_la(x, mode):
    return x["log_alpha"] if mode == "kda" else x["la_s"]


@pytest.mark.parametrize("mode", ["kda", "gdn"])
@pytest.mark.parametrize("T", [64, 200])
def test_reduced_forward_equals_expanded_and_oracle(mode, T):
    import gated_delta_rule_gdn2_b200 as g
    x = reduced_inputs(2, T, 3, 128, 128, mode, "bf16", seed=610 + T)
    q, k, v = (dev(x[n], "bf16") for n in ("q", "k", "v"))
    S0 = dev_state(x["S0"])
    o, ST = g.chunk_fwd_reduced(q, k, v, dev(reduced_la(x, mode), "bf16"), dev(x["beta"], "bf16"), mode, S0=S0)
    o_e, ST_e = g.chunk_fwd(*[dev(x[n], "bf16") for n in NAMES], S0=S0)
    assert g.gdn2_get_device_status() == 0
    np.testing.assert_array_equal(host(o), host(o_e))
    np.testing.assert_array_equal(host(ST), host(ST_e))
    o_ref, ST_ref = oracle.fwd(*[x[n] for n in NAMES], x["S0"])
    check("o", host(o), o_ref, TOL_BF16)
    check("S_T", host(ST), ST_ref, TOL_BF16)


@pytest.mark.parametrize("mode", ["kda", "gdn"])
def test_reduced_forward_fp32_mode(mode):
    import gated_delta_rule_gdn2_b200 as g
    x = reduced_inputs(2, 100, 2, 64, 128, mode, "fp32", seed=71)
    q, k, v = (dev(x[n], "fp32") for n in ("q", "k", "v"))
    o, ST = g.chunk_fwd_reduced(q, k, v, dev(reduced_la(x, mode), "fp32"), dev(x["beta"], "fp32"), mode,
                                S0=dev_state(x["S0"]))
    assert g.gdn2_get_device_status() == 0
    o_ref, ST_ref = oracle.fwd(*[x[n] for n in NAMES], x["S0"])
    check("o", host(o), o_ref, TOL_FP32)
    check("S_T", host(ST), ST_ref, TOL_FP32)


@pytest.mark.parametrize("mode", ["kda", "gdn"])
@pytest.mark.parametrize("B,T,H", [(2, 150, 2), (2, 1024, 4)])
def test_reduced_backward_matches_oracle(mode, B, T, H):
    import gated_delta_rule_gdn2_b200 as g
    x = reduced_inputs(B, T, H, 128, 128, mode, "bf16", seed=820 + T)
    rng = np.random.default_rng(T)
    dST = (0.1 * rng.standard_normal(x["S0"].shape)).astype(np.float32)
    q, k, v = (dev(x[n], "bf16") for n in ("q", "k", "v"))
    S0 = dev_state(x["S0"])
    dO = dev(x["dO"], "bf16")
    gr = g.chunk_bwd_reduced(q, k, v, dev(reduced_la(x, mode), "bf16"), dev(x["beta"], "bf16"), S0, dO,
                             dev_state(dST), mode=mode)
    ge = g.chunk_bwd(*[dev(x[n], "bf16") for n in NAMES], S0, dO, dev_state(dST))
    assert g.gdn2_get_device_status() == 0
    # the gradients that do not pass through a gate reduction: the general call's bits
    for n in ("dq", "dk", "dv", "dS0") + (("dlog_alpha",) if mode == "kda" else ()):
        np.testing.assert_array_equal(host(gr[n]), host(ge[n]))
    # against the oracle: these gates push the largest gradient entries to ~15,
    # so entries are held to the per-element bound 5e-2 + 2^-7 |ref| (rel-L2 <= 1e-2)
    ref = oracle.bwd(*[x[n] for n in NAMES], x["S0"], x["dO"], dST)
    for n in ("dq", "dk", "dv", "dS0"):
        check(n, host(gr[n]), ref[n], TOL_BF16_ELEM)
    check_sum("dbeta", host(gr["dbeta"]), ref["db"].sum(-1) + ref["dw"].sum(-1),
              np.abs(ref["db"]).sum(-1) + np.abs(ref["dw"]).sum(-1))
    if mode == "kda":
        check("dlog_alpha", host(gr["dlog_alpha"]), ref["dlog_alpha"], TOL_BF16_ELEM)
    else:
        check_sum("dlog_alpha", host(gr["dlog_alpha"]), ref["dlog_alpha"].sum(-1),
                  np.abs(ref["dlog_alpha"]).sum(-1))


@pytest.mark.parametrize("mode", ["kda", "gdn"])
@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 128, 128), ("fp32", 64, 128), ("bf16", 128, 64)])
def test_reduced_decode_equals_expanded(mode, dtype, dk, dv):
    import gated_delta_rule_gdn2_b200 as g
    B, H = 4, 3
    S = dev_state(0.02 * np.random.default_rng(1).standard_normal((B, H, dk, dv)).astype(np.float32))
    S_e = S.clone()
    Sref = host(S)
    for step in range(8):
        x = reduced_inputs(B, 1, H, dk, dv, mode, dtype, seed=900 + step)
        x1 = {n: v[:, 0] for n, v in x.items() if n not in ("S0",)}
        o = g.decode_step_reduced(*(dev(x1[n], dtype) for n in ("q", "k", "v")), dev(reduced_la(x1, mode), dtype),
                                  dev(x1["beta"], dtype), S, mode=mode)
        o_e = g.decode_step(*[dev(x1[n], dtype) for n in NAMES], S_e)
        o_ref, Sref = oracle.decode(*[x1[n] for n in NAMES], Sref)
        np.testing.assert_array_equal(host(o), host(o_e))
        check("o step %d" % step, host(o), o_ref, TOL_BF16 if dtype == "bf16" else TOL_FP32)
    assert g.gdn2_get_device_status() == 0
    np.testing.assert_array_equal(host(S), host(S_e))


def test_reduced_unsupported_combinations():
    import gated_delta_rule_gdn2_b200 as g
    x = reduced_inputs(1, 64, 1, 64, 64, "kda", "bf16", seed=1)
    q, k, v = (dev(x[n], "bf16") for n in ("q", "k", "v"))
    with pytest.raises(g.Gdn2Error) as e:
        g.chunk_fwd_reduced(q, k, v, dev(x["log_alpha"], "bf16"), dev(x["beta"], "bf16"), "kda")
    assert e.value.status == -2
