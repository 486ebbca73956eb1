/*
 * Plain fp64 CPU oracle of the layer pieces around the Gated DeltaNet-2
 * mixer: the input prologue and the output epilogue, with their backward
 * passes.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test-suite uses it.  It shares no code, header or
 * constant with the CUDA library.
 *
 * What it computes ("Why NVIDIA Gated DeltaNet-2 separates erase and write
 * gates" (axbrief), section on implications for practitioners: the query and
 * key paths are a linear projection, a short causal convolution, SiLU and L2
 * normalisation; the value path a projection, a short convolution and SiLU;
 * the output an RMS normalisation and a SiLU output gate.  The projections
 * are matrix products outside this library; the gate activations follow the
 * recurrence's definitions alpha = exp(log_alpha) in (0, 1), b, w in [0, 1]):
 *
 *   conv   y[t,c] = sum_{j=0}^{K-1} W[c][j] x[t-(K-1)+j, c]   (x before t = 0 is 0)
 *   SiLU   s = y sigmoid(y)
 *   L2     q = s / sqrt(sum_c s^2 + eps)                      (per token and head)
 *   gates  log_alpha = -log(1 + e^{-x_a}),  b = sigmoid(x_b),  w = sigmoid(x_w)
 *   RMS    z = o / sqrt(mean_j o_j^2 + eps) * gamma[j] * silu(g_j)
 *
 * Readings where the page is silent: the convolution is depthwise (one filter
 * of K taps per channel of each head, weights [H*D][K]) and causal within a
 * sequence; eps = 1e-6 in both normalisations; the RMS weight gamma [dv] is
 * shared by the heads.  The backward passes are the hand-derived vector-
 * Jacobian products of exactly these lines.
 *
 * Layouts: token tensors [B,T,H,D] contiguous; doubles throughout.
 */
#include <math.h>
#include <stddef.h>
#include <string.h>

#define NORM_EPS 1e-6

static inline size_t at(int b, int t, int h, int T, int H, int D) { return (((size_t)b * T + t) * H + h) * (size_t)D; }

static inline double sigm(double x) { return 1.0 / (1.0 + exp(-x)); }

/* conv + SiLU of one tensor: y (pre-activation) and s = silu(y) */
static void conv_silu(const double *x, const double *W, int K, double *y, double *s, int B, int T, int H, int D)
{
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int h = 0; h < H; ++h)
                for (int c = 0; c < D; ++c) {
                    const double *w = W + ((size_t)h * D + c) * K;
                    double acc = 0.0;
                    for (int j = 0; j < K; ++j) {
                        const int tt = t - (K - 1) + j;
                        if (tt >= 0) acc += w[j] * x[at(b, tt, h, T, H, D) + c];
                    }
                    const size_t o = at(b, t, h, T, H, D) + c;
                    y[o] = acc;
                    s[o] = acc * sigm(acc);
                }
}

/* Prologue forward of one path.  l2: normalise over the D channels (q, k). */
void oracle_prologue_path(const double *x, const double *W, int K, double *out, int B, int T, int H, int D,
                          int l2, double *y_work, double *s_work)
{
    conv_silu(x, W, K, y_work, s_work, B, T, H, D);
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int h = 0; h < H; ++h) {
                const size_t o = at(b, t, h, T, H, D);
                double n = 1.0;
                if (l2) {
                    double ss = 0.0;
                    for (int c = 0; c < D; ++c) ss += s_work[o + c] * s_work[o + c];
                    n = sqrt(ss + NORM_EPS);
                }
                for (int c = 0; c < D; ++c) out[o + c] = s_work[o + c] / n;
            }
}

/* Prologue backward of one path: dout -> dx and dW (dW accumulated over
 * every batch and token). */
void oracle_prologue_path_bwd(const double *x, const double *W, int K, const double *dout, double *dx, double *dW,
                              int B, int T, int H, int D, int l2, double *y_work, double *s_work, double *dy_work)
{
    conv_silu(x, W, K, y_work, s_work, B, T, H, D);
    /* through the L2 norm and the SiLU: dy */
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int h = 0; h < H; ++h) {
                const size_t o = at(b, t, h, T, H, D);
                double n = 1.0, dot = 0.0;
                if (l2) {
                    double ss = 0.0;
                    for (int c = 0; c < D; ++c) ss += s_work[o + c] * s_work[o + c];
                    n = sqrt(ss + NORM_EPS);
                    /* out = s / n:  ds = (dout - out (out . dout)) / n */
                    for (int c = 0; c < D; ++c) dot += (s_work[o + c] / n) * dout[o + c];
                }
                for (int c = 0; c < D; ++c) {
                    const double out = s_work[o + c] / n;
                    const double ds = (dout[o + c] - (l2 ? out * dot : 0.0)) / n;
                    const double y = y_work[o + c], sg = sigm(y);
                    dy_work[o + c] = ds * sg * (1.0 + y * (1.0 - sg));
                }
            }
    /* through the convolution */
    memset(dx, 0, sizeof(double) * (size_t)B * T * H * D);
    memset(dW, 0, sizeof(double) * (size_t)H * D * K);
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int h = 0; h < H; ++h)
                for (int c = 0; c < D; ++c) {
                    const double dy = dy_work[at(b, t, h, T, H, D) + c];
                    const double *w = W + ((size_t)h * D + c) * K;
                    double *dw = dW + ((size_t)h * D + c) * K;
                    for (int j = 0; j < K; ++j) {
                        const int tt = t - (K - 1) + j;
                        if (tt < 0) continue;
                        dx[at(b, tt, h, T, H, D) + c] += w[j] * dy;
                        dw[j] += x[at(b, tt, h, T, H, D) + c] * dy;
                    }
                }
}

/* Gate activations, elementwise over n values: kind 0 log_alpha, 1 sigmoid. */
void oracle_gate(const double *x, double *out, size_t n, int kind)
{
    for (size_t i = 0; i < n; ++i) out[i] = kind == 0 ? -log1p(exp(-x[i])) : sigm(x[i]);
}

/* ... and their backward: d log_alpha / dx = 1 - sigmoid(x); d sigmoid / dx = s (1 - s). */
void oracle_gate_bwd(const double *x, const double *dout, double *dx, size_t n, int kind)
{
    for (size_t i = 0; i < n; ++i) {
        const double s = sigm(x[i]);
        dx[i] = dout[i] * (kind == 0 ? 1.0 - s : s * (1.0 - s));
    }
}

/* Epilogue forward: z = o / rms(o) * gamma * silu(g) per token and head. */
void oracle_epilogue(const double *o, const double *g, const double *gamma, double *z, int B, int T, int H, int D)
{
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int h = 0; h < H; ++h) {
                const size_t p = at(b, t, h, T, H, D);
                double ss = 0.0;
                for (int j = 0; j < D; ++j) ss += o[p + j] * o[p + j];
                const double r = 1.0 / sqrt(ss / D + NORM_EPS);
                for (int j = 0; j < D; ++j) z[p + j] = o[p + j] * r * gamma[j] * g[p + j] * sigm(g[p + j]);
            }
}

/* Epilogue backward: dz -> do, dg, dgamma (dgamma summed over batches, tokens
 * and heads). */
void oracle_epilogue_bwd(const double *o, const double *g, const double *gamma, const double *dz, double *dO,
                         double *dg, double *dgamma, int B, int T, int H, int D)
{
    memset(dgamma, 0, sizeof(double) * (size_t)D);
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int h = 0; h < H; ++h) {
                const size_t p = at(b, t, h, T, H, D);
                double ss = 0.0;
                for (int j = 0; j < D; ++j) ss += o[p + j] * o[p + j];
                const double r = 1.0 / sqrt(ss / D + NORM_EPS);
                /* z = n gamma silu(g), n = o r:  dn = dz gamma silu(g);
                 * do = r (dn - n mean(n dn)) */
                double m = 0.0;
                for (int j = 0; j < D; ++j) {
                    const double gg = g[p + j], sg = sigm(gg), n = o[p + j] * r;
                    const double dn = dz[p + j] * gamma[j] * gg * sg;
                    m += n * dn;
                    dgamma[j] += dz[p + j] * n * gg * sg;
                    dg[p + j] = dz[p + j] * n * gamma[j] * sg * (1.0 + gg * (1.0 - sg));
                }
                m /= D;
                for (int j = 0; j < D; ++j) {
                    const double gg = g[p + j], sg = sigm(gg), n = o[p + j] * r;
                    const double dn = dz[p + j] * gamma[j] * gg * sg;
                    dO[p + j] = r * (dn - n * m);
                }
            }
}
