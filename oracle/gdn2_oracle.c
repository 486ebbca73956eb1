/*
 * Plain fp64 CPU oracle of the Gated DeltaNet-2 sequence mixer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header or constant with
 * the CUDA library.
 *
 * What it computes (per batch b, head h, token t = 1..T):
 *
 *   "Why NVIDIA Gated DeltaNet-2 separates erase and write gates" (axbrief),
 *   section "Gated Delta Rule-2: per-channel erase/write split", recurrence:
 *
 *       S_t = (I - k_t (b_t . k_t)^T) D_t S_{t-1} + k_t (w_t . v_t)^T,
 *       D_t = Diag(alpha_t),  alpha_t = exp(log_alpha_t),
 *
 *   with S_t in R^{dk x dv} (rows = key channels, columns = value channels),
 *   erase gate b_t in [0,1]^dk on the key axis and write gate w_t in [0,1]^dv
 *   on the value axis (same section, gate definitions).  The readout is the
 *   post-update o_t = S_t^T q_t (the pages leave it open; this is the reading
 *   the build fixes).  Evaluated literally, with the decayed state
 *   S' = D_t S_{t-1} read by the erase:
 *
 *       S'  = D_t S_{t-1}
 *       u   = w_t . v_t - S'^T (b_t . k_t)
 *       S_t = S' + k_t u^T
 *       o_t = S_t^T q_t
 *
 *   The backward pass is the reverse-time adjoint of exactly these four
 *   lines ("gate-aware vector-Jacobian product", same page and section): with
 *   Shat = dL/dS_t,
 *
 *       Shat += q_t do_t^T            dq_t = S_t do_t
 *       du    = Shat^T k_t            dk_t = Shat u
 *       dw_t  = du . v_t              dv_t = du . w_t
 *       dg    = -S' du                db_t = dg . k_t,  dk_t += dg . b_t
 *       dS'   = Shat - g du^T         dla_t[c] = sum_j dS'[c,j] S'[c,j]
 *       Shat  = D_t dS'   (-> dL/dS_{t-1})
 *
 *   States needed in reverse are replayed from fp64 checkpoints taken every
 *   64 tokens.
 *
 * Layouts: token tensors [B,T,H,D] contiguous (D fastest); state
 * [B,H,dk,dv] row-major.  All arrays are double.  Heads are independent and
 * run under OpenMP.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define CKPT 64

static inline size_t tok_index(int b, int t, int h, int T, int H, int D)
{
    return (((size_t)b * T + t) * H + h) * (size_t)D;
}

/* One token of the recurrence on one head, in place.  Sp receives S' (the
 * decayed state) when non-null; u receives the residual edit when non-null. */
static void step(double *S, const double *q, const double *k, const double *v,
                 const double *la, const double *bg, const double *wg,
                 double *o, double *Sp_out, double *u_out, int dk, int dv,
                 double *u)
{
    /* S' = D S */
    for (int c = 0; c < dk; ++c) {
        double a = exp(la[c]);
        double *row = S + (size_t)c * dv;
        for (int j = 0; j < dv; ++j) row[j] *= a;
    }
    if (Sp_out) memcpy(Sp_out, S, sizeof(double) * (size_t)dk * dv);
    /* u = w.v - S'^T (b.k) */
    for (int j = 0; j < dv; ++j) u[j] = wg[j] * v[j];
    for (int c = 0; c < dk; ++c) {
        double g = bg[c] * k[c];
        const double *row = S + (size_t)c * dv;
        for (int j = 0; j < dv; ++j) u[j] -= g * row[j];
    }
    if (u_out) memcpy(u_out, u, sizeof(double) * (size_t)dv);
    /* S = S' + k u^T */
    for (int c = 0; c < dk; ++c) {
        double *row = S + (size_t)c * dv;
        for (int j = 0; j < dv; ++j) row[j] += k[c] * u[j];
    }
    /* o = S^T q */
    if (o) {
        for (int j = 0; j < dv; ++j) o[j] = 0.0;
        for (int c = 0; c < dk; ++c) {
            const double *row = S + (size_t)c * dv;
            for (int j = 0; j < dv; ++j) o[j] += q[c] * row[j];
        }
    }
}

/* Forward over T tokens.  S0 may be NULL (zero state); S_T may be NULL. */
void oracle_fwd(const double *q, const double *k, const double *v,
                const double *la, const double *bg, const double *wg,
                const double *S0, double *o, double *S_T,
                int B, int T, int H, int dk, int dv)
{
    const size_t sz = (size_t)dk * dv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        int b = bh / H, h = bh % H;
        double *S = (double *)malloc(sizeof(double) * sz);
        double *u = (double *)malloc(sizeof(double) * dv);
        if (S0) memcpy(S, S0 + (size_t)bh * sz, sizeof(double) * sz);
        else memset(S, 0, sizeof(double) * sz);
        for (int t = 0; t < T; ++t) {
            size_t ik = tok_index(b, t, h, T, H, dk);
            size_t iv = tok_index(b, t, h, T, H, dv);
            step(S, q + ik, k + ik, v + iv, la + ik, bg + ik, wg + iv,
                 o + iv, NULL, NULL, dk, dv, u);
        }
        if (S_T) memcpy(S_T + (size_t)bh * sz, S, sizeof(double) * sz);
        free(u);
        free(S);
    }
}

/* One decode step: tokens [B,H,D], state [B,H,dk,dv] updated in place. */
void oracle_decode(const double *q, const double *k, const double *v,
                   const double *la, const double *bg, const double *wg,
                   double *S, double *o, int B, int H, int dk, int dv)
{
    const size_t sz = (size_t)dk * dv;
#pragma omp parallel for schedule(static)
    for (int bh = 0; bh < B * H; ++bh) {
        double *u = (double *)malloc(sizeof(double) * dv);
        size_t ik = (size_t)bh * dk, iv = (size_t)bh * dv;
        step(S + (size_t)bh * sz, q + ik, k + ik, v + iv, la + ik, bg + ik,
             wg + iv, o + iv, NULL, NULL, dk, dv, u);
        free(u);
    }
}

/* Reverse-time backward.  Gradients of L = sum_t <do_t, o_t> + <dS_T, S_T>
 * with respect to q, k, v, log_alpha, b, w and S0.  S0 and dS_T may be NULL
 * (zero); dS0 may be NULL (not returned). */
void oracle_bwd(const double *q, const double *k, const double *v,
                const double *la, const double *bg, const double *wg,
                const double *S0, const double *dO, const double *dS_T,
                double *dq, double *dk_, double *dv_, double *dla,
                double *db, double *dw, double *dS0,
                int B, int T, int H, int dk, int dv)
{
    const size_t sz = (size_t)dk * dv;
    const int nseg = (T + CKPT - 1) / CKPT;
#pragma omp parallel for schedule(dynamic, 1)
    for (int bh = 0; bh < B * H; ++bh) {
        int b = bh / H, h = bh % H;
        double *ck = (double *)malloc(sizeof(double) * sz * (size_t)(nseg + 1));
        double *Sall = (double *)malloc(sizeof(double) * sz * (CKPT + 1));
        double *Spall = (double *)malloc(sizeof(double) * sz * CKPT);
        double *uall = (double *)malloc(sizeof(double) * (size_t)dv * CKPT);
        double *Sh = (double *)malloc(sizeof(double) * sz);
        double *dSp = (double *)malloc(sizeof(double) * sz);
        double *u = (double *)malloc(sizeof(double) * dv);
        double *du = (double *)malloc(sizeof(double) * dv);
        double *dg = (double *)malloc(sizeof(double) * dk);

        /* forward pass keeping a checkpoint at every segment start */
        double *S = Sall;
        if (S0) memcpy(S, S0 + (size_t)bh * sz, sizeof(double) * sz);
        else memset(S, 0, sizeof(double) * sz);
        for (int t = 0; t < T; ++t) {
            if (t % CKPT == 0) memcpy(ck + (size_t)(t / CKPT) * sz, S, sizeof(double) * sz);
            size_t ik = tok_index(b, t, h, T, H, dk);
            size_t iv = tok_index(b, t, h, T, H, dv);
            step(S, q + ik, k + ik, v + iv, la + ik, bg + ik, wg + iv,
                 NULL, NULL, NULL, dk, dv, u);
        }

        if (dS_T) memcpy(Sh, dS_T + (size_t)bh * sz, sizeof(double) * sz);
        else memset(Sh, 0, sizeof(double) * sz);

        for (int seg = nseg - 1; seg >= 0; --seg) {
            int t0 = seg * CKPT;
            int t1 = t0 + CKPT < T ? t0 + CKPT : T;
            /* replay the segment: Sall[i] = state after token t0+i-1 */
            memcpy(Sall, ck + (size_t)seg * sz, sizeof(double) * sz);
            for (int t = t0; t < t1; ++t) {
                int i = t - t0;
                memcpy(Sall + (size_t)(i + 1) * sz, Sall + (size_t)i * sz, sizeof(double) * sz);
                size_t ik = tok_index(b, t, h, T, H, dk);
                size_t iv = tok_index(b, t, h, T, H, dv);
                step(Sall + (size_t)(i + 1) * sz, q + ik, k + ik, v + iv, la + ik,
                     bg + ik, wg + iv, NULL, Spall + (size_t)i * sz,
                     uall + (size_t)i * dv, dk, dv, u);
            }
            for (int t = t1 - 1; t >= t0; --t) {
                int i = t - t0;
                size_t ik = tok_index(b, t, h, T, H, dk);
                size_t iv = tok_index(b, t, h, T, H, dv);
                const double *St = Sall + (size_t)(i + 1) * sz;
                const double *Sp = Spall + (size_t)i * sz;
                const double *ut = uall + (size_t)i * dv;
                const double *qt = q + ik, *kt = k + ik, *lat = la + ik, *bt = bg + ik;
                const double *vt = v + iv, *wt = wg + iv, *dot = dO + iv;
                /* o_t = S_t^T q_t */
                for (int c = 0; c < dk; ++c) {
                    double *row = Sh + (size_t)c * dv;
                    const double *srow = St + (size_t)c * dv;
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        row[j] += qt[c] * dot[j];
                        acc += srow[j] * dot[j];
                    }
                    dq[ik + c] = acc;
                }
                /* S_t = S' + k u^T */
                for (int j = 0; j < dv; ++j) du[j] = 0.0;
                for (int c = 0; c < dk; ++c) {
                    const double *row = Sh + (size_t)c * dv;
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        du[j] += row[j] * kt[c];
                        acc += row[j] * ut[j];
                    }
                    dk_[ik + c] = acc;
                }
                /* u = w.v - S'^T g */
                for (int j = 0; j < dv; ++j) {
                    dw[iv + j] = du[j] * vt[j];
                    dv_[iv + j] = du[j] * wt[j];
                }
                for (int c = 0; c < dk; ++c) {
                    const double *sprow = Sp + (size_t)c * dv;
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) acc += sprow[j] * du[j];
                    dg[c] = -acc;
                }
                /* g = b.k */
                for (int c = 0; c < dk; ++c) {
                    db[ik + c] = dg[c] * kt[c];
                    dk_[ik + c] += dg[c] * bt[c];
                }
                /* dS' = Shat - g du^T ; dla = rowsum(dS' . S') ; Shat = D dS' */
                for (int c = 0; c < dk; ++c) {
                    double g = bt[c] * kt[c];
                    double a = exp(lat[c]);
                    const double *row = Sh + (size_t)c * dv;
                    const double *sprow = Sp + (size_t)c * dv;
                    double *drow = dSp + (size_t)c * dv;
                    double acc = 0.0;
                    for (int j = 0; j < dv; ++j) {
                        drow[j] = row[j] - g * du[j];
                        acc += drow[j] * sprow[j];
                    }
                    dla[ik + c] = acc;
                    double *out = Sh + (size_t)c * dv;
                    for (int j = 0; j < dv; ++j) out[j] = a * drow[j];
                }
            }
        }
        if (dS0) memcpy(dS0 + (size_t)bh * sz, Sh, sizeof(double) * sz);
        free(dg); free(du); free(u); free(dSp); free(Sh);
        free(uall); free(Spall); free(Sall); free(ck);
    }
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
