"""GPU parity of gdn2_chunk_fwd against the fp64 oracle on identical seeded
inputs, through the C ABI: bf16 tensor-core path (rel-L2 <= 1e-2, max-abs <=
5e-2 on o and S_T) and fp32 precision mode (rel-L2 <= 1e-4)."""
import numpy as np
import pytest

import oracle
from gpu_util import TOL_BF16, TOL_FP32, NAMES, check, dev_state, host, sub_heads, tokens
from gated_delta_rule_gdn2_b200.inputs import WORKLOADS, make_inputs, make_workload

pytestmark = pytest.mark.gpu


def run_fwd(x, dtype, with_state=True):
    import gated_delta_rule_gdn2_b200 as g
    o, ST = g.chunk_fwd(*tokens(x, dtype), S0=dev_state(x["S0"]), output_final_state=with_state)
    assert g.gdn2_get_device_status() == 0
    return host(o), (host(ST) if ST is not None else None)


def oracle_fwd(x):
    return oracle.fwd(*[x[n] for n in NAMES], x["S0"])


@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200, 320])
def test_bf16_matches_oracle(dk, dv, T):
    x = make_inputs(2, T, 3, dk, dv, seed=100 + T + dk + 2 * dv, dtype="bf16")
    o, ST = run_fwd(x, "bf16")
    o_ref, ST_ref = oracle_fwd(x)
    check("o", o, o_ref, TOL_BF16)
    check("S_T", ST, ST_ref, TOL_BF16)


def test_bf16_zero_initial_state_and_no_final_state():
    x = make_inputs(1, 130, 2, 128, 128, seed=3, dtype="bf16", s0_std=0.0)
    o, ST = run_fwd(x, "bf16")
    o_ref, ST_ref = oracle_fwd(x)
    check("o", o, o_ref, TOL_BF16)
    check("S_T", ST, ST_ref, TOL_BF16)
    o2, none = run_fwd(x, "bf16", with_state=False)
    assert none is None
    np.testing.assert_array_equal(o2, o)


@pytest.mark.parametrize("scale", [8.0, 40.0])
def test_bf16_fast_decay_takes_exact_path(scale):
    """Decays far outside the pages' range: some chunks span more than e^-64 in
    a key channel (the exact slow path) and the rest do not."""
    x = make_inputs(2, 256, 2, 128, 128, seed=9, dtype="bf16")
    rng = np.random.default_rng(1)
    la = x["log_alpha"]
    mask = rng.random(la.shape) < 0.05
    la[mask] = -scale * rng.random(mask.sum()).astype(np.float32)
    from gated_delta_rule_gdn2_b200.inputs import round_bf16
    x["log_alpha"] = round_bf16(la)
    o, ST = run_fwd(x, "bf16")
    o_ref, ST_ref = oracle_fwd(x)
    check("o", o, o_ref, TOL_BF16)
    check("S_T", ST, ST_ref, TOL_BF16)


def test_bf16_reset():
    x = make_inputs(1, 150, 2, 128, 128, seed=10, dtype="bf16")
    x["log_alpha"][:] = -800.0
    o, ST = run_fwd(x, "bf16")
    o_ref, ST_ref = oracle_fwd(x)
    check("o", o, o_ref, TOL_BF16)
    check("S_T", ST, ST_ref, TOL_BF16)


def test_fp32_mode_tiny_workload():
    w = WORKLOADS["tiny_fp32"]
    x = make_workload(w)
    o, ST = run_fwd(x, "fp32")
    o_ref, ST_ref = oracle_fwd(x)
    check("o", o, o_ref, TOL_FP32)
    check("S_T", ST, ST_ref, TOL_FP32)


@pytest.mark.parametrize("T", [1, 100, 257])
def test_fp32_mode_shapes(T):
    x = make_inputs(2, T, 2, 128, 64, seed=T, dtype="fp32")
    o, ST = run_fwd(x, "fp32")
    o_ref, ST_ref = oracle_fwd(x)
    check("o", o, o_ref, TOL_FP32)
    check("S_T", ST, ST_ref, TOL_FP32)


def test_empty_sequence_copies_state():
    import torch
    import gated_delta_rule_gdn2_b200 as g
    x = make_inputs(2, 0, 2, 64, 64, seed=1, dtype="bf16")
    o, ST = g.chunk_fwd(*tokens(x, "bf16"), S0=dev_state(x["S0"]))
    assert o.shape == (2, 0, 2, 64)
    np.testing.assert_array_equal(host(ST), x["S0"])
    e = [torch.empty((1, 0, 1, 64), device="cuda", dtype=torch.bfloat16) for _ in range(6)]
    _, ST0 = g.chunk_fwd(*e)
    assert float(ST0.abs().max()) == 0.0


def test_deterministic_and_segment_invariant():
    """Bitwise run-to-run determinism; processing T in two segments (S_T of the
    first as S0 of the second) agrees with one pass."""
    import gated_delta_rule_gdn2_b200 as g
    x = make_inputs(2, 320, 2, 128, 128, seed=12, dtype="bf16")
    o1, S1 = run_fwd(x, "bf16")
    o2, S2 = run_fwd(x, "bf16")
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(S1, S2)
    xa = {n: (v[:, :128] if n != "S0" else v) for n, v in x.items()}
    xb = {n: (v[:, 128:] if n != "S0" else None) for n, v in x.items()}
    oa, Sa = g.chunk_fwd(*tokens(xa, "bf16"), S0=dev_state(x["S0"]))
    ob, Sb = g.chunk_fwd(*tokens(xb, "bf16"), S0=Sa)
    o_cat = np.concatenate([host(oa), host(ob)], axis=1)
    check("o", o_cat, o1, TOL_BF16)
    check("S_T", host(Sb), S1, TOL_BF16)


def _sampled_full(w, T=None, heads=((0, 0), (3, 7), (7, 15))):
    x = make_workload(w, T)
    o, ST = run_fwd(x, "bf16")
    xs = sub_heads(x, list(heads))
    o_ref, ST_ref = oracle_fwd(xs)
    for i, (b, h) in enumerate(heads):
        check("o[%d,:,%d]" % (b, h), o[b, :, h], o_ref[i, :, 0], TOL_BF16)
        check("S_T[%d,%d]" % (b, h), ST[b, h], ST_ref[i, 0], TOL_BF16)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(ST))


def test_prefill_full_size_sampled_heads():
    """B=8, T=4096, H=16, d=128 (the 1.3B layer shape), in the benchmark's
    launch configuration; the oracle recomputes three whole heads."""
    _sampled_full(WORKLOADS["prefill"])


@pytest.mark.parametrize("T", [8192, 32768, 131072])
def test_long_sequence_sampled_heads(T):
    _sampled_full(WORKLOADS["long"], T=T, heads=((0, 0), (0, 11)))


@pytest.mark.parametrize("dk", [128, 64])
def test_segmented_and_one_cta_per_sequence(dk):
    """B1 H4 T4096: with the workspace gdn2_chunk_fwd_workspace asks for, the
    forward runs four sequence segments side by side; given only the plain
    B*H*64*dk*4 bytes it runs one CTA per sequence.  Both against the oracle,
    and against each other."""
    import torch
    import gated_delta_rule_gdn2_b200 as g
    B, T, H = 1, 4096, 4
    x = make_inputs(B, T, H, dk, dk, seed=404 + dk, dtype="bf16")
    toks = tokens(x, "bf16")
    S0 = dev_state(x["S0"])
    plain = B * H * 64 * dk * 4
    full = g.gdn2_chunk_fwd_workspace(B, T, H, dk, dk, g.GDN2_BF16)
    assert full > plain
    outs = []
    for nbytes in (full, plain):
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        o = torch.empty((B, T, H, dk), dtype=torch.bfloat16, device="cuda")
        ST = torch.empty((B, H, dk, dk), dtype=torch.float32, device="cuda")
        st = g.gdn2_chunk_fwd(*toks, S0, o, ST, B, T, H, dk, dk, g.GDN2_BF16, ws, nbytes,
                              torch.cuda.current_stream().cuda_stream)
        assert st == 0
        assert g.gdn2_get_device_status() == 0
        outs.append((host(o), host(ST)))
    o_ref, ST_ref = oracle_fwd(x)
    for o, ST in outs:
        check("o", o, o_ref, TOL_BF16)
        check("S_T", ST, ST_ref, TOL_BF16)
    check("o segmented vs one CTA per sequence", outs[0][0], outs[1][0], TOL_BF16)


@pytest.mark.parametrize("B,T,H", [(2, 1088, 16), (1, 3264, 16), (1, 4096, 3)])
def test_segmented_uneven_segments(B, T, H):
    """The segment path at shapes whose chunk count does not divide evenly
    (17 chunks in 2 segments; 51 in 5; 64 in 8 with three heads), with a
    nonzero S0 (the first segment starts from it, the others are corrected
    from their scanned start states): against the oracle and against the
    one-CTA-per-sequence path."""
    import torch
    import gated_delta_rule_gdn2_b200 as g
    x = make_inputs(B, T, H, 128, 128, seed=T + B + H, dtype="bf16")
    toks = tokens(x, "bf16")
    S0 = dev_state(x["S0"])
    plain = B * H * 64 * 128 * 4
    full = g.gdn2_chunk_fwd_workspace(B, T, H, 128, 128, g.GDN2_BF16)
    assert full > plain
    outs = []
    for nbytes in (full, plain):
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        o = torch.empty((B, T, H, 128), dtype=torch.bfloat16, device="cuda")
        ST = torch.empty((B, H, 128, 128), dtype=torch.float32, device="cuda")
        assert g.gdn2_chunk_fwd(*toks, S0, o, ST, B, T, H, 128, 128, g.GDN2_BF16, ws, nbytes) == 0
        assert g.gdn2_get_device_status() == 0
        outs.append((host(o), host(ST)))
    heads = [(0, 0), (B - 1, H - 1)]
    xs = sub_heads(x, heads)
    o_ref, ST_ref = oracle_fwd(xs)
    for o, ST in outs:
        for i, (b, h) in enumerate(heads):
            check("o[%d,:,%d]" % (b, h), o[b, :, h], o_ref[i, :, 0], TOL_BF16)
            check("S_T[%d,%d]" % (b, h), ST[b, h], ST_ref[i, 0], TOL_BF16)
    check("o segmented vs one CTA per sequence", outs[0][0], outs[1][0], TOL_BF16)
    check("S_T segmented vs one CTA per sequence", outs[0][1], outs[1][1], TOL_BF16)
