"""numpy restatement of the CUDA chunk algorithm -- a diagnostic, not the oracle.

It follows the kernels step for step (64-token chunks, decays referenced to
the chunk boundary, the WY solve, the inter-chunk update) so that
the chunk algebra can be checked against the token-by-token oracle on the CPU,
and, with ``bf16=True``, rounds every tensor-core operand to bfloat16 where the
kernel does, which estimates the error budget of the bf16 path.

Chunk algebra for one chunk with start state S (rows r, i = 0..Cn-1, per key
channel c; L = in-chunk cumulative log-decay):
    A[r,i] = sum_c (b_r k_r)[c] k_i[c] e^{L_r[c]-L_i[c]}   (i < r)
    M[r,i] = sum_c q_r[c] k_i[c] e^{L_r[c]-L_i[c]}          (i <= r)
    T = (I + A)^{-1},  W = T (g e^{L}),  Uv = T (w v)
    U = Uv - W S,  O = (q e^{L}) S + M U,  S' = e^{L_end} S + (k e^{L_end - L})^T U
Every decay factor is referenced to the chunk start (see chunk_fwd_head for
the guard that keeps the one factor above 1 in range).
"""
from __future__ import annotations

import numpy as np

C = 64


def rnd_bf16(x):
    x32 = np.asarray(x, dtype=np.float32)
    u = x32.view(np.uint32).astype(np.uint64)
    r = (((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16).astype(np.uint32)
    return r.view(np.float32).astype(np.float64)


SPAN_GUARD = 64.0


def chunk_fwd_head(q, k, v, la, b, w, S0, bf16=False, force_slow=False):
    """One head: q, k, la, b [T, dk]; v, w [T, dv]; S0 [dk, dv] -> (o [T, dv], S_T).

    Fast path (chunk decay span <= SPAN_GUARD in every key channel): all decay
    factors are referenced to the chunk start,
        Gt = g e^{L}, Qt = q e^{L} (in (0,1]),  Kb = k e^{-L} (<= e^{span}),
        [A; M] = [Gt; Qt] Kb^T,   S' = Diag(e^{L_end}) (S + Kb^T U).
    Slow path (a chunk whose decay span exceeds the guard): A and M from
    e^{L_r - L_i} term by term and S' = Diag(e^{L_end}) S + (k e^{L_end-L})^T U.
    """
    rd = rnd_bf16 if bf16 else (lambda x: np.asarray(x, dtype=np.float64))
    T, dk = q.shape
    dv = v.shape[1]
    S = np.array(S0, dtype=np.float64)
    o = np.zeros((T, dv))
    for n0 in range(0, T, C):
        n1 = min(T, n0 + C)
        Cn = n1 - n0
        qc, kc, vc, lac, bc, wc = (x[n0:n1].astype(np.float64) for x in (q, k, v, la, b, w))
        L = np.cumsum(lac, axis=0)
        g = bc * kc
        Gt = g * np.exp(L)
        Qt = qc * np.exp(L)
        WV = wc * vc
        gam = np.exp(L[-1])
        slow = force_slow or np.max(-L[-1]) > SPAN_GUARD
        if not slow:
            Kb = kc * np.exp(-L)
            A = rd(Gt) @ rd(Kb).T
            M = rd(Qt) @ rd(Kb).T
        else:
            A = np.zeros((Cn, Cn))
            M = np.zeros((Cn, Cn))
            for r in range(Cn):
                for i in range(r + 1):
                    e = np.exp(L[r] - L[i])
                    A[r, i] = np.sum(g[r] * kc[i] * e)
                    M[r, i] = np.sum(qc[r] * kc[i] * e)
        A = np.tril(A, -1)
        M = np.tril(M, 0)
        Tm = np.linalg.inv(np.eye(Cn) + A)
        W = rd(Tm) @ rd(Gt)
        Uv = rd(Tm) @ rd(WV)
        U = Uv - rd(W) @ rd(S)
        o[n0:n1] = rd(Qt) @ rd(S) + rd(M) @ rd(U)
        if not slow:
            S = gam[:, None] * (S + rd(Kb).T @ rd(U))
        else:
            Kt = kc * np.exp(L[-1] - L)
            S = gam[:, None] * S + rd(Kt).T @ rd(U)
    return o, S


def chunk_fwd(q, k, v, la, b, w, S0=None, bf16=False, force_slow=False):
    """Token tensors [B,T,H,D]; returns (o, S_T) like oracle.fwd."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    for bb in range(B):
        for h in range(H):
            s0 = np.zeros((dk, dv)) if S0 is None else S0[bb, h]
            o[bb, :, h], ST[bb, h] = chunk_fwd_head(q[bb, :, h], k[bb, :, h], v[bb, :, h],
                                                    la[bb, :, h], b[bb, :, h], w[bb, :, h], s0, bf16,
                                                    force_slow)
    return o, ST


def chunk_bwd_head(q, k, v, la, b, w, S0, dO, dST, bf16=False, opts=()):
    """Backward of chunk_fwd_head (fast path only), rounding the tensor-core
    operands where the CUDA backward rounds them.  Returns dict of gradients."""
    rd = rnd_bf16 if bf16 else (lambda x: np.asarray(x, dtype=np.float64))
    out_rd = rd if "fp32_out" not in opts else (lambda x: np.asarray(x, dtype=np.float64))
    T, dk = q.shape
    dv = v.shape[1]
    # forward states at chunk boundaries (bf16 as the state pass stores them)
    S = np.array(S0, dtype=np.float64)
    states = [rd(S)]
    for n0 in range(0, T, C):
        n1 = min(T, n0 + C)
        _, S = chunk_fwd_head(q[n0:n1], k[n0:n1], v[n0:n1], la[n0:n1], b[n0:n1], w[n0:n1], S, bf16)
        states.append(rd(S))
    g = {n: np.zeros((T, dk)) for n in ("dq", "dk", "dlog_alpha", "db")}
    g.update({n: np.zeros((T, dv)) for n in ("dv", "dw")})
    dS = np.zeros((dk, dv)) if dST is None else np.array(dST, dtype=np.float64)
    nchunks = (T + C - 1) // C
    for n in range(nchunks - 1, -1, -1):
        n0, n1 = n * C, min(T, n * C + C)
        Sn = states[n]
        Snext = states[n + 1]
        qc, kc, vc, lac, bc, wc, dOc = (x[n0:n1].astype(np.float64) for x in (q, k, v, la, b, w, dO))
        L = np.cumsum(lac, axis=0)
        gg = bc * kc
        e, ie = np.exp(L), np.exp(-L)
        Gt, Qt, Kb, WV = rd(gg * e), rd(qc * e), rd(kc * ie), rd(wc * vc)
        gam = np.exp(L[-1])
        A = np.tril(Gt @ Kb.T, -1)
        M = np.tril(Qt @ Kb.T, 0)
        Tm = rd(np.linalg.inv(np.eye(n1 - n0) + A))
        Mb = rd(M)
        W = rd(-(Tm @ Gt))
        Uv = Tm @ WV
        U = rd(Uv + W @ Sn)
        Dh = rd(gam[:, None] * dS)
        rs = np.sum(dS * Snext, axis=1)
        dU = rd(Mb.T @ dOc + Kb @ Dh)
        dRHS = Tm.T @ dU
        nR = rd(-dRHS)
        g["dv"][n0:n1] = out_rd(-nR * wc)  # the kernel forms dv, dw from the bf16 -dRHS tile
        g["dw"][n0:n1] = out_rd(-nR * vc)
        dKb = U @ Dh.T
        dMm = np.tril(dOc @ U.T, 0)
        dAm = np.tril(nR @ U.T, -1)
        dMdiag = np.diag(dMm).copy()  # the kernel keeps the diagonal out of the Gram products
        dMm = dMm - np.diag(dMdiag)
        dMb, dAb = rd(dMm), rd(dAm)
        dQt = dOc @ Sn.T + dMb @ Kb
        dGt = nR @ Sn.T + dAb @ Kb
        dKb = dKb + dAb.T @ Gt + dMb.T @ Qt
        dS = gam[:, None] * dS + Qt.T @ dOc + Gt.T @ nR
        dq = dQt * e
        dg = dGt * e
        dkk = dKb * ie
        dL = dQt * qc * e + dGt * gg * e - dKb * kc * ie
        dq += dMdiag[:, None] * kc
        dkk += dMdiag[:, None] * qc
        dL[-1] += rs
        g["dq"][n0:n1] = out_rd(dq)
        g["dk"][n0:n1] = out_rd(dkk + dg * bc)
        g["db"][n0:n1] = out_rd(dg * kc)
        g["dlog_alpha"][n0:n1] = out_rd(np.cumsum(dL[::-1], axis=0)[::-1])
    g["dS0"] = dS
    return g


def chunk_bwd(q, k, v, la, b, w, S0, dO, dST=None, bf16=False, opts=()):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = {n: np.zeros((B, T, H, dk)) for n in ("dq", "dk", "dlog_alpha", "db")}
    out.update({n: np.zeros((B, T, H, dv)) for n in ("dv", "dw")})
    out["dS0"] = np.zeros((B, H, dk, dv))
    for bb in range(B):
        for h in range(H):
            s0 = np.zeros((dk, dv)) if S0 is None else S0[bb, h]
            dst = None if dST is None else dST[bb, h]
            r = chunk_bwd_head(q[bb, :, h], k[bb, :, h], v[bb, :, h], la[bb, :, h], b[bb, :, h],
                               w[bb, :, h], s0, dO[bb, :, h], dst, bf16, opts)
            for n in out:
                if n == "dS0":
                    out[n][bb, h] = r[n]
                else:
                    out[n][bb, :, h] = r[n]
    return out
