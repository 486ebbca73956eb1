"""Pins of the fp64 oracle against facts the pages and the mathematics fix.

None of these re-types the oracle's own update: each check reaches the answer
by another route (explicit transition matrices, a textbook special case, a
closed form, an invariant, a hand-worked example, finite differences, or
linearity).  The last group plants mistakes in copies of the oracle and checks
that some pin fails for each.

Method source: "Why NVIDIA Gated DeltaNet-2 separates erase and write gates"
(axbrief), section "Gated Delta Rule-2: per-channel erase/write split".
"""
import json
import os

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def rand_case(rng, B=1, T=6, H=1, dk=3, dv=4, la_scale=1.0, s0=True):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    la = -la_scale * np.abs(rng.standard_normal((B, T, H, dk)))
    b = rng.random((B, T, H, dk))
    w = rng.random((B, T, H, dv))
    S0 = rng.standard_normal((B, H, dk, dv)) if s0 else None
    return q, k, v, la, b, w, S0


def brute_force(q, k, v, la, b, w, S0):
    """Unrolled transition products.  For each head, build the dk x dk matrices
    A_t = (I - k_t (b_t . k_t)^T) Diag(alpha_t) and form
        S_t = A_t ... A_1 S_0 + sum_{s<=t} A_t ... A_{s+1} k_s (w_s . v_s)^T
    directly from the pages' recurrence, then o_t = S_t^T q_t."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    for bb in range(B):
        for h in range(H):
            A = []
            X = []
            for t in range(T):
                kt = k[bb, t, h]
                At = (np.eye(dk) - np.outer(kt, b[bb, t, h] * kt)) @ np.diag(np.exp(la[bb, t, h]))
                A.append(At)
                X.append(np.outer(kt, w[bb, t, h] * v[bb, t, h]))
            s0 = np.zeros((dk, dv)) if S0 is None else S0[bb, h]
            for t in range(T):
                P = np.eye(dk)
                for s in range(t, -1, -1):
                    P = P @ A[s]
                St = P @ s0
                for s in range(t + 1):
                    P = np.eye(dk)
                    for r in range(t, s, -1):
                        P = P @ A[r]
                    St = St + P @ X[s]
                o[bb, t, h] = St.T @ q[bb, t, h]
                if t == T - 1:
                    ST[bb, h] = St
    return o, ST


# --------------------------------------------------------------------------
# forward pins


@pytest.mark.parametrize("T", [1, 2, 5, 8])
def test_brute_force_transition_products(T):
    rng = np.random.default_rng(10 + T)
    args = rand_case(rng, B=2, T=T, H=2, dk=3, dv=4)
    o, ST = oracle.fwd(*args)
    o_ref, ST_ref = brute_force(*args)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-13)
    np.testing.assert_allclose(ST, ST_ref, rtol=0, atol=1e-13)


def test_hand_worked_example():
    g = json.load(open(os.path.join(HERE, "golden", "hand_worked_T2.json")))
    inp = g["inputs"]
    sh = lambda x: np.array(x, dtype=np.float64)[None, :, None, :]
    o, ST = oracle.fwd(sh(inp["q"]), sh(inp["k"]), sh(inp["v"]), np.log(sh(inp["alpha"])),
                       sh(inp["b"]), sh(inp["w"]), np.array(inp["S0"])[None, None])
    np.testing.assert_allclose(o[0, :, 0], np.array(g["expected"]["o"]), atol=1e-14)
    np.testing.assert_allclose(ST[0, 0], np.array(g["expected"]["S_T"]), atol=1e-14)


def test_reduces_to_kda():
    """b = w = beta (scalar per token, broadcast) gives Kimi Delta Attention:
    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T."""
    rng = np.random.default_rng(3)
    q, k, v, la, _, _, S0 = rand_case(rng, B=1, T=7, H=2, dk=4, dv=3)
    beta = rng.random((1, 7, 2, 1))
    o, ST = oracle.fwd(q, k, v, la, np.broadcast_to(beta, q.shape),
                       np.broadcast_to(beta, v.shape), S0)
    for h in range(2):
        S = S0[0, h].copy()
        for t in range(7):
            kt, bt = k[0, t, h], beta[0, t, h, 0]
            S = (np.eye(4) - bt * np.outer(kt, kt)) @ np.diag(np.exp(la[0, t, h])) @ S \
                + bt * np.outer(kt, v[0, t, h])
            np.testing.assert_allclose(o[0, t, h], S.T @ q[0, t, h], atol=1e-13)
        np.testing.assert_allclose(ST[0, h], S, atol=1e-13)


def test_reduces_to_gated_deltanet():
    """Additionally a scalar decay a_t: S_t = a_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T."""
    rng = np.random.default_rng(4)
    q, k, v, _, _, _, S0 = rand_case(rng, B=1, T=7, H=1, dk=4, dv=5)
    beta = rng.random((1, 7, 1, 1))
    a = rng.uniform(0.2, 1.0, (1, 7, 1, 1))
    o, ST = oracle.fwd(q, k, v, np.broadcast_to(np.log(a), q.shape),
                       np.broadcast_to(beta, q.shape), np.broadcast_to(beta, v.shape), S0)
    S = S0[0, 0].copy()
    for t in range(7):
        kt, bt = k[0, t, 0], beta[0, t, 0, 0]
        S = a[0, t, 0, 0] * (np.eye(4) - bt * np.outer(kt, kt)) @ S + bt * np.outer(kt, v[0, t, 0])
        np.testing.assert_allclose(o[0, t, 0], S.T @ q[0, t, 0], atol=1e-13)
    np.testing.assert_allclose(ST[0, 0], S, atol=1e-13)


def test_exact_erase_projection():
    """b = 1, alpha = 1, unit k: the edit replaces what the state returns for
    k_t, so S_t^T k_t = w_t . v_t exactly (delta rule with L2-normalised keys,
    laonpeople Gated DeltaNet page, 'precise eraser' principle)."""
    rng = np.random.default_rng(5)
    dk, dv, T = 6, 5, 20
    k = rng.standard_normal((1, 1, dk))
    S = rng.standard_normal((1, 1, dk, dv))
    for t in range(T):
        kt = rng.standard_normal((1, 1, dk))
        kt /= np.linalg.norm(kt)
        vt = rng.standard_normal((1, 1, dv))
        wt = rng.random((1, 1, dv))
        qt = rng.standard_normal((1, 1, dk))
        _, S = oracle.decode(qt, kt, vt, np.zeros((1, 1, dk)), np.ones((1, 1, dk)), wt, S)
        np.testing.assert_allclose(S[0, 0].T @ kt[0, 0], wt[0, 0] * vt[0, 0], atol=1e-12)
    del k


def test_no_erase_closed_form():
    """b = 0: S_T = Diag(e^{L_T}) S_0 + sum_t Diag(e^{L_T - L_t}) k_t (w_t . v_t)^T
    with L_t the cumulative log-decay; o_t = S_t^T q_t with the same sum to t."""
    rng = np.random.default_rng(6)
    q, k, v, la, _, w, S0 = rand_case(rng, B=1, T=9, H=1, dk=4, dv=3)
    o, ST = oracle.fwd(q, k, v, la, np.zeros_like(q), w, S0)
    L = np.cumsum(la[0, :, 0], axis=0)
    for t in range(9):
        St = np.exp(L[t])[:, None] * S0[0, 0]
        for s in range(t + 1):
            St = St + np.exp(L[t] - L[s])[:, None] * np.outer(k[0, s, 0], w[0, s, 0] * v[0, s, 0])
        np.testing.assert_allclose(o[0, t, 0], St.T @ q[0, t, 0], atol=1e-13)
    np.testing.assert_allclose(ST[0, 0], St, atol=1e-13)


def test_reset():
    """log_alpha = -800: the decayed state is exactly zero, so S_t = k_t (w_t . v_t)^T."""
    rng = np.random.default_rng(7)
    q, k, v, _, b, w, S0 = rand_case(rng, B=1, T=5, H=1, dk=4, dv=3)
    o, ST = oracle.fwd(q, k, v, np.full(q.shape, -800.0), b, w, S0)
    for t in range(5):
        St = np.outer(k[0, t, 0], w[0, t, 0] * v[0, t, 0])
        np.testing.assert_allclose(o[0, t, 0], St.T @ q[0, t, 0], atol=1e-15)
    np.testing.assert_allclose(ST[0, 0], St, atol=1e-15)


def test_decode_matches_forward_token_by_token():
    rng = np.random.default_rng(8)
    q, k, v, la, b, w, S0 = rand_case(rng, B=2, T=6, H=3, dk=4, dv=5)
    o, ST = oracle.fwd(q, k, v, la, b, w, S0)
    S = S0.copy()
    for t in range(6):
        ot, S = oracle.decode(q[:, t], k[:, t], v[:, t], la[:, t], b[:, t], w[:, t], S)
        np.testing.assert_allclose(ot, o[:, t], atol=1e-14)
    np.testing.assert_allclose(S, ST, atol=1e-14)


def test_zero_state_and_empty_sequence():
    rng = np.random.default_rng(9)
    q, k, v, la, b, w, _ = rand_case(rng, B=1, T=4, H=2, dk=3, dv=3)
    o1, S1 = oracle.fwd(q, k, v, la, b, w, None)
    o2, S2 = oracle.fwd(q, k, v, la, b, w, np.zeros((1, 2, 3, 3)))
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(S1, S2)
    S0 = rng.standard_normal((1, 2, 3, 3))
    e = np.zeros((1, 0, 2, 3))
    o, ST = oracle.fwd(e, e, e, e, e, e, S0)
    assert o.shape == (1, 0, 2, 3)
    np.testing.assert_array_equal(ST, S0)


# --------------------------------------------------------------------------
# backward pins


def _loss(args, dO, dST):
    o, ST = oracle.fwd(*args)
    return float(np.sum(o * dO) + np.sum(ST * dST))


def test_backward_central_differences():
    """Every gradient (q, k, v, log_alpha, b, w, S0) against central finite
    differences of L = sum <dO, o> + <dS_T, S_T> at B=1, T=16, H=1, dk=dv=8."""
    rng = np.random.default_rng(11)
    args = list(rand_case(rng, B=1, T=16, H=1, dk=8, dv=8, la_scale=0.3))
    dO = rng.standard_normal(args[2].shape)
    dST = rng.standard_normal(args[6].shape)
    g = oracle.bwd(*args, dO, dST)
    names = ["dq", "dk", "dv", "dlog_alpha", "db", "dw", "dS0"]
    h = 1e-6
    for i, name in enumerate(names):
        x = args[i]
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            keep = x[idx]
            x[idx] = keep + h
            lp = _loss(args, dO, dST)
            x[idx] = keep - h
            lm = _loss(args, dO, dST)
            x[idx] = keep
            fd[idx] = (lp - lm) / (2 * h)
        err = np.linalg.norm(fd - g[name]) / np.linalg.norm(fd)
        assert err < 1e-6, (name, err)


def test_backward_adjoint_identity():
    """o and S_T are jointly linear in (S0, v); hence
    <dO, o(dS0', dv')> + <dS_T, S_T(dS0', dv')> = <dS0, dS0'> + <dv, dv'> exactly."""
    rng = np.random.default_rng(12)
    q, k, v, la, b, w, S0 = rand_case(rng, B=2, T=70, H=2, dk=5, dv=4, la_scale=0.2)
    dO = rng.standard_normal(v.shape)
    dST = rng.standard_normal(S0.shape)
    g = oracle.bwd(q, k, v, la, b, w, S0, dO, dST)
    o, ST = oracle.fwd(q, k, v, la, b, w, S0)
    lhs = np.sum(dO * o) + np.sum(dST * ST)
    rhs = np.sum(g["dS0"] * S0) + np.sum(g["dv"] * v)
    assert abs(lhs - rhs) < 1e-11 * max(1.0, abs(lhs))


def test_backward_no_upstream_state_gradient():
    rng = np.random.default_rng(13)
    q, k, v, la, b, w, S0 = rand_case(rng, B=1, T=3, H=1, dk=3, dv=3)
    dO = rng.standard_normal(v.shape)
    g1 = oracle.bwd(q, k, v, la, b, w, S0, dO, None)
    g2 = oracle.bwd(q, k, v, la, b, w, S0, dO, np.zeros_like(S0))
    for n in g1:
        np.testing.assert_array_equal(g1[n], g2[n])


# --------------------------------------------------------------------------
# planted mistakes: each edited copy of the oracle must fail some pin above

MUTANTS = {
    # readout from the state before this token's edit
    "readout_before_update": ("    /* o = S^T q */\n    if (o) {",
                              "    for (int c = 0; c < dk; ++c) {\n"
                              "        double *row = S + (size_t)c * dv;\n"
                              "        for (int j = 0; j < dv; ++j) row[j] -= k[c] * u[j];\n    }\n"
                              "    if (o) {"),
    # erase gate applied on the write side instead of the read side
    "gate_wrong_side": ("        double g = bg[c] * k[c];\n        const double *row = S + (size_t)c * dv;\n"
                        "        for (int j = 0; j < dv; ++j) u[j] -= g * row[j];",
                        "        double g = k[c];\n        const double *row = S + (size_t)c * dv;\n"
                        "        for (int j = 0; j < dv; ++j) u[j] -= g * row[j];"),
    # write gate dropped
    "write_gate_dropped": ("u[j] = wg[j] * v[j];", "u[j] = v[j];"),
    # key read with q instead of k
    "erase_reads_q": ("double g = bg[c] * k[c];\n        const double *row = S + (size_t)c * dv;\n"
                      "        for (int j = 0; j < dv; ++j) u[j] -= g * row[j];",
                      "double g = bg[c] * q[c];\n        const double *row = S + (size_t)c * dv;\n"
                      "        for (int j = 0; j < dv; ++j) u[j] -= g * row[j];"),
    # sign of the erase-side gradient flipped
    "bwd_dg_sign": ("dg[c] = -acc;", "dg[c] = acc;"),
    # gate factor missing inside the dk inner product
    "bwd_gate_missing_in_dk": ("dk_[ik + c] += dg[c] * bt[c];", "dk_[ik + c] += dg[c];"),
    # decay gradient taken against the undecayed state
    "bwd_dla_wrong_state": ("acc += drow[j] * sprow[j];", "acc += drow[j] * sprow[j] / a;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = oracle.source_text()
    assert src.count(old) == 1, name
    bad = oracle.compile_variant(src.replace(old, new), str(tmp_path / ("m_%s.so" % name)))
    rng = np.random.default_rng(21)
    args = list(rand_case(rng, B=1, T=5, H=1, dk=3, dv=3, la_scale=0.5))
    caught = []
    o, ST = bad.fwd(*args)
    o_ref, ST_ref = brute_force(*args)
    caught.append(not (np.allclose(o, o_ref, atol=1e-10) and np.allclose(ST, ST_ref, atol=1e-10)))
    dO = rng.standard_normal(args[2].shape)
    dST = rng.standard_normal(args[6].shape)
    g = bad.bwd(*args, dO, dST)
    h = 1e-6
    for i, gname in enumerate(["dq", "dk", "dv", "dlog_alpha", "db", "dw", "dS0"]):
        x = args[i]
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            keep = x[idx]
            x[idx] = keep + h
            o1, s1 = bad.fwd(*args)
            x[idx] = keep - h
            o2, s2 = bad.fwd(*args)
            x[idx] = keep
            fd[idx] = (np.sum((o1 - o2) * dO) + np.sum((s1 - s2) * dST)) / (2 * h)
        caught.append(np.linalg.norm(fd - g[gname]) > 1e-5 * np.linalg.norm(fd))
    assert any(caught), name
