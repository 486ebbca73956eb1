"""The chunk algorithm of the CUDA path, restated in numpy (tests/emu_chunk.py),
against the token-by-token oracle on the CPU: exact in fp64 on both the fast
(chunk-boundary pivot) and the slow (term-by-term decay) path, for ragged
chunks, fast decays and resets; and within the bf16 tolerance when every
tensor-core operand is rounded to bfloat16 where the kernels round it."""
import numpy as np
import pytest

import emu_chunk as E
import oracle
from gated_delta_rule_gdn2_b200.inputs import make_inputs


def _args(x):
    return [x[n] for n in ("q", "k", "v", "log_alpha", "b", "w")] + [x["S0"]]


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
@pytest.mark.parametrize("slow", [False, True])
def test_chunk_algebra_exact(T, slow):
    x = make_inputs(1, T, 2, 64, 64, seed=T, dtype="fp32")
    o, S = oracle.fwd(*_args(x))
    oe, Se = E.chunk_fwd(*_args(x), force_slow=slow)
    np.testing.assert_allclose(oe, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Se, S, rtol=0, atol=1e-12)


def test_chunk_algebra_guard_and_reset():
    x = make_inputs(1, 150, 1, 64, 64, seed=7, dtype="fp32")
    la = x["log_alpha"]
    la[0, 70:76, 0, :4] = -40.0  # one chunk spans e^-240 in four channels: slow path
    o, S = oracle.fwd(*_args(x))
    oe, Se = E.chunk_fwd(*_args(x))
    np.testing.assert_allclose(oe, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Se, S, rtol=0, atol=1e-12)
    la[:] = -800.0
    o, S = oracle.fwd(*_args(x))
    oe, Se = E.chunk_fwd(*_args(x))
    np.testing.assert_allclose(oe, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(Se, S, rtol=0, atol=1e-12)


def test_bf16_error_budget():
    x = make_inputs(1, 512, 2, 128, 128, seed=1001, dtype="bf16")
    o, S = oracle.fwd(*_args(x))
    oe, Se = E.chunk_fwd(*_args(x), bf16=True)
    rel = lambda a, b: np.linalg.norm(a - b) / np.linalg.norm(b)
    assert rel(oe, o) < 5e-3 and rel(Se, S) < 5e-3


@pytest.mark.parametrize("T", [1, 64, 150])
def test_chunk_backward_algebra_exact(T):
    """The backward's chunk algebra (as the CUDA reverse pass computes it) is
    the oracle's gradient in fp64."""
    x = make_inputs(1, T, 2, 64, 64, seed=T, dtype="fp32", with_do=True)
    rng = np.random.default_rng(T)
    dST = rng.standard_normal(x["S0"].shape)
    ref = oracle.bwd(*_args(x), x["dO"], dST)
    got = E.chunk_bwd(*_args(x), x["dO"], dST)
    for n in ref:
        np.testing.assert_allclose(got[n], ref[n], rtol=0, atol=1e-11)


def test_chunk_backward_bf16_error_budget():
    x = make_inputs(1, 512, 1, 128, 128, seed=1004, dtype="bf16", with_do=True)
    ref = oracle.bwd(*_args(x), x["dO"], None)
    got = E.chunk_bwd(*_args(x), x["dO"], None, bf16=True)
    rel = lambda a, b: np.linalg.norm(a - b) / np.linalg.norm(b)
    for n in ref:
        assert rel(got[n], ref[n]) < 8e-3, n
        assert np.max(np.abs(got[n] - ref[n])) < 5e-2, n


def test_segment_composition_exact():
    """The state update is affine in the state, so a sequence cut into segments
    composes from each segment's end state from a zero start (S_loc) and from
    an identity start with the write term w . v removed (the transition Phi):
    S_start(p) = Phi(p-1) S_start(p-1) + S_loc(p-1), and each segment's o from
    its true start state equals the whole sequence's o (the sequence-segmented
    forward's algebra, checked on the oracle in fp64)."""
    B, T, H, dk, dv, P = 1, 48, 2, 8, 8, 4
    x = make_inputs(B, T, H, dk, dv, seed=21, dtype="fp32")
    o_full, S_full = oracle.fwd(x["q"], x["k"], x["v"], x["log_alpha"], x["b"], x["w"], x["S0"])
    L = T // P
    seg = lambda a, p: a[:, p * L:(p + 1) * L]
    eye = np.broadcast_to(np.eye(dk), (B, H, dk, dk)).copy()
    S = x["S0"].astype(np.float64)
    for p in range(P):
        toks = [seg(x[n], p) for n in ("q", "k", "v", "log_alpha", "b", "w")]
        _, S_loc = oracle.fwd(*toks, None)
        zeros = np.zeros_like(toks[2])
        _, Phi = oracle.fwd(toks[0], toks[1], zeros, toks[3], toks[4], zeros, eye)
        o_seg, S_end = oracle.fwd(*toks, S)
        np.testing.assert_allclose(o_seg, seg(o_full, p), rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(S_end, np.einsum("bhij,bhjk->bhik", Phi, S) + S_loc, rtol=1e-11, atol=1e-12)
        S = S_end
    np.testing.assert_allclose(S, S_full, rtol=1e-11, atol=1e-12)


def test_backward_segment_composition_exact():
    """The reverse chain composes over segments with the transpose of the
    forward's segment transition: the state gradient at a segment's start is
    Phi^T (its gradient at the segment's end) + the segment's own contribution
    (its dS0 for a zero end gradient), and each segment's backward from its true
    start state and end gradient gives the whole sequence's gradients on that
    segment (the algebra a segmented backward would rest on, on the oracle in
    fp64)."""
    B, T, H, dk, dv, P = 1, 48, 2, 8, 8, 4
    x = make_inputs(B, T, H, dk, dv, seed=23, dtype="fp32", with_do=True)
    rng = np.random.default_rng(9)
    dST = rng.standard_normal((B, H, dk, dv))
    names = ("q", "k", "v", "log_alpha", "b", "w")
    full = oracle.bwd(*[x[n] for n in names], x["S0"], x["dO"], dST)
    L = T // P
    seg = lambda a, p: a[:, p * L:(p + 1) * L]
    eye = np.broadcast_to(np.eye(dk), (B, H, dk, dk)).copy()
    # start states of the segments (forward) and their transitions
    starts, phis = [x["S0"].astype(np.float64)], []
    for p in range(P):
        toks = [seg(x[n], p) for n in names]
        zeros = np.zeros_like(toks[2])
        phis.append(oracle.fwd(toks[0], toks[1], zeros, toks[3], toks[4], zeros, eye)[1])
        starts.append(oracle.fwd(*toks, starts[-1])[1])
    # the reverse scan over segments, then each segment's gradients
    dS_end = dST
    for p in reversed(range(P)):
        toks = [seg(x[n], p) for n in names]
        loc = oracle.bwd(*toks, starts[p], seg(x["dO"], p), np.zeros_like(dST))["dS0"]
        dS_start = np.einsum("bhji,bhjk->bhik", phis[p], dS_end) + loc
        g = oracle.bwd(*toks, starts[p], seg(x["dO"], p), dS_end)
        np.testing.assert_allclose(g["dS0"], dS_start, rtol=1e-10, atol=1e-11)
        for n in ("dq", "dk", "dv", "dlog_alpha", "db", "dw"):
            np.testing.assert_allclose(g[n], seg(full[n], p), rtol=1e-10, atol=1e-11)
        dS_end = dS_start
    np.testing.assert_allclose(dS_end, full["dS0"], rtol=1e-10, atol=1e-11)
