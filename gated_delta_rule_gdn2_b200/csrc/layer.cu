// The layer pieces around the mixer, as single fused kernels: the input
// prologue (short causal convolution, SiLU and L2 norm of the query and key
// paths, convolution and SiLU of the value path, and the gate activations)
// and the output epilogue (RMS norm with a SiLU output gate), each with its
// backward pass.
//
// "Why NVIDIA Gated DeltaNet-2 separates erase and write gates" (axbrief),
// section on implications for practitioners: the query/key path is a linear
// projection, a short causal convolution, SiLU and L2 normalisation; the
// value path a projection, a short convolution and SiLU; the output an RMS
// normalisation and a SiLU output gate.  (The projections are matrix products
// outside this library.)  The convolution is depthwise and causal within a
// sequence: y[t, c] = sum_j W[c][j] x[t - (K-1) + j, c], taps before the
// sequence's first token reading zero; eps = 1e-6 in both norms; the RMS
// weight gamma [dv] is shared by the heads.  Gates: log_alpha = log
// sigmoid(x_a), b = sigmoid(x_b), w = sigmoid(x_w).
//
// Layout of the work: one warp walks 8 consecutive token rows of one head;
// lanes hold D/32 channels each, so every row access is one coalesced
// D-element read or write and a row's reductions (the L2 norm, the RMS) are
// warp shuffles.  The convolution keeps a sliding window of the last K input
// rows in registers, so each input element is read from memory once.  The
// backward recomputes the forward of each row, runs the convolution's
// transpose with a window of K pending rows, and sums the filter gradient per
// CTA; a second kernel adds the CTAs' sums in a fixed order (deterministic).
// All of it is bandwidth-bound elementwise and stencil work: no tensor cores.
#include "common.cuh"
#include "gdn2.h"
#include "launch.h"

namespace gdn2 {
namespace layer {

constexpr int kRowsPerWarp = 8, kWarps = 8, kRowsPerCta = kRowsPerWarp * kWarps;
constexpr int kMaxConv = 4;
constexpr float kEps = 1e-6f;

__device__ __forceinline__ float sigm(float x) { return 1.f / (1.f + __expf(-x)); }

// CPL consecutive elements of a row at p (this lane's channels) as fp32 ...
template <typename T, int CPL>
__device__ __forceinline__ void ld(const T *p, float (&v)[CPL]) {
    if constexpr (sizeof(T) == 2 && CPL == 4) {
        const uint2 u = *reinterpret_cast<const uint2 *>(p);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
        v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
    } else if constexpr (sizeof(T) == 2 && CPL == 2) {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
        v[0] = a.x; v[1] = a.y;
    } else if constexpr (CPL == 4) {
        const float4 a = *reinterpret_cast<const float4 *>(p);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    } else {
        const float2 a = *reinterpret_cast<const float2 *>(p);
        v[0] = a.x; v[1] = a.y;
    }
}
// ... and back.
template <typename T, int CPL>
__device__ __forceinline__ void st(T *p, const float (&v)[CPL]) {
    if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int i = 0; i < CPL; i += 2)
            *reinterpret_cast<__nv_bfloat162 *>(p + i) = __floats2bfloat162_rn(v[i], v[i + 1]);
    } else if constexpr (CPL == 4) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    } else {
        *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
    }
}

// The sequence that holds token row r: [start, end).  Fixed-length batches
// (cu == nullptr): sequences of T rows; packed: the offsets cu[0..N].
struct SeqCursor {
    const int *cu;
    int N, T;
    int s;  // packed: the current sequence
    long start, end;
    __device__ __forceinline__ void seek(long r) {
        if (!cu) {
            start = r - r % T;
            end = start + T;
            return;
        }
        int lo = 0, hi = N - 1;  // the last s with cu[s] <= r
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (cu[mid] <= r) lo = mid; else hi = mid - 1;
        }
        s = lo;
        while (s + 1 < N && cu[s + 1] <= r) ++s;
        start = cu[s];
        end = cu[s + 1];
    }
    // advance to row r >= the current row
    __device__ __forceinline__ void advance(long r) {
        if (r < end) return;
        if (!cu) { seek(r); return; }
        while (s + 1 < N && cu[s + 1] <= r) ++s;
        start = cu[s];
        end = cu[s + 1];
    }
};

struct PrologueArgs {
    const void *xq, *xk, *xv, *xa, *xb, *xw;  // pre-activations [rows][H][D]
    const float *Wq, *Wk, *Wv;                // filters [H * D][K]
    void *q, *k, *v, *la, *b, *w;             // mixer inputs [rows][H][D]
    long rows;
    int H, K, T;                              // T: tokens per sequence of a fixed-length batch
    const int *cu;                            // packed: N + 1 offsets (or nullptr)
    int N;
};

// The forward of one convolution path over this warp's rows.
template <typename Tin, int D, int K>
__device__ __forceinline__ void conv_path_fwd(const Tin *x, const float *W, Tin *out, bool l2, long r0, int nr, int h, int H,
                              SeqCursor cur, int lane) {
    constexpr int CPL = D / 32;
    const int c0 = lane * CPL;
    float wt[K][CPL], win[K][CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i)
#pragma unroll
        for (int j = 0; j < K; ++j) wt[j][i] = W[((size_t)h * D + c0 + i) * K + j];
    cur.seek(r0);
#pragma unroll
    for (int j = 0; j < K - 1; ++j) {  // the rows before r0 that the window reaches, in r0's sequence
        const long r = r0 - (K - 1) + j;
        if (r >= cur.start && r >= 0) ld<Tin, CPL>(x + ((size_t)r * H + h) * D + c0, win[j]);
        else
#pragma unroll
            for (int i = 0; i < CPL; ++i) win[j][i] = 0.f;
    }
    for (int it = 0; it < nr; ++it) {
        const long r = r0 + it;
        cur.advance(r);
        if (r == cur.start)  // a sequence starts here: nothing before it reaches in
#pragma unroll
            for (int j = 0; j < K - 1; ++j)
#pragma unroll
                for (int i = 0; i < CPL; ++i) win[j][i] = 0.f;
        ld<Tin, CPL>(x + ((size_t)r * H + h) * D + c0, win[K - 1]);
        float s[CPL], ss = 0.f;
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            float y = 0.f;
#pragma unroll
            for (int j = 0; j < K; ++j) y = fmaf(wt[j][i], win[j][i], y);
            s[i] = y * sigm(y);
            ss = fmaf(s[i], s[i], ss);
        }
        if (l2) {
            const float n = rsqrtf(warp_sum(ss) + kEps);
#pragma unroll
            for (int i = 0; i < CPL; ++i) s[i] *= n;
        }
        st<Tin, CPL>(out + ((size_t)r * H + h) * D + c0, s);
#pragma unroll
        for (int j = 0; j < K - 1; ++j)
#pragma unroll
            for (int i = 0; i < CPL; ++i) win[j][i] = win[j + 1][i];
    }
}

template <typename Tin, int D>
__device__ __forceinline__ void gate_rows_fwd(const Tin *x, Tin *out, bool logsig, long r0, int nr, int h, int H, int lane) {
    constexpr int CPL = D / 32;
    for (int it = 0; it < nr; ++it) {
        const size_t o = ((size_t)(r0 + it) * H + h) * D + lane * CPL;
        float v[CPL];
        ld<Tin, CPL>(x + o, v);
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            // log sigmoid(x) = -log(1 + e^{-x}), kept accurate for large |x|
            v[i] = logsig ? (v[i] < 0.f ? v[i] - log1pf(__expf(v[i])) : -log1pf(__expf(-v[i]))) : sigm(v[i]);
        }
        st<Tin, CPL>(out + o, v);
    }
}

template <typename Tin, int DK, int DV, int K>
__global__ void __launch_bounds__(kWarps * 32) prologue_fwd_kernel(PrologueArgs a) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, h = blockIdx.y;
    const long r0 = (long)blockIdx.x * kRowsPerCta + warp * kRowsPerWarp;
    if (r0 >= a.rows) return;
    const int nr = (int)min((long)kRowsPerWarp, a.rows - r0);
    SeqCursor cur{a.cu, a.N, a.T, 0, 0, 0};
    conv_path_fwd<Tin, DK, K>(static_cast<const Tin *>(a.xq), a.Wq, static_cast<Tin *>(a.q), true, r0, nr, h, a.H,
                              cur, lane);
    conv_path_fwd<Tin, DK, K>(static_cast<const Tin *>(a.xk), a.Wk, static_cast<Tin *>(a.k), true, r0, nr, h, a.H,
                              cur, lane);
    conv_path_fwd<Tin, DV, K>(static_cast<const Tin *>(a.xv), a.Wv, static_cast<Tin *>(a.v), false, r0, nr, h, a.H,
                              cur, lane);
    gate_rows_fwd<Tin, DK>(static_cast<const Tin *>(a.xa), static_cast<Tin *>(a.la), true, r0, nr, h, a.H, lane);
    gate_rows_fwd<Tin, DK>(static_cast<const Tin *>(a.xb), static_cast<Tin *>(a.b), false, r0, nr, h, a.H, lane);
    gate_rows_fwd<Tin, DV>(static_cast<const Tin *>(a.xw), static_cast<Tin *>(a.w), false, r0, nr, h, a.H, lane);
}

// ---------------------------------------------------------------------------
// Prologue backward

struct PrologueBwdArgs {
    PrologueArgs f;                         // inputs as the forward's (its outputs unused)
    const void *dq, *dk, *dv, *dla, *db, *dw;  // gradients of the mixer inputs
    void *dxq, *dxk, *dxv, *dxa, *dxb, *dxw;   // gradients of the pre-activations
    float *part;                            // per CTA filter-gradient sums [grid.x][H][dk + dk + dv][K]
};

// One convolution path's backward over this warp's rows: dx for its own rows
// (from dy of rows up to K - 1 further, in the same sequence) and this warp's
// sum of the filter gradient into red[c][j] (shared, per warp slot).
template <typename Tin, int D, int K>
__device__ __forceinline__ void conv_path_bwd(const Tin *x, const float *W, const Tin *dout, Tin *dx, bool l2, long r0, int nr,
                              long rows, int h, int H, SeqCursor cur, int lane, float (*dW)[K]) {
    constexpr int CPL = D / 32;
    const int c0 = lane * CPL;
    float wt[K][CPL], win[K][CPL], pend[K][CPL], gw[K][CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i)
#pragma unroll
        for (int j = 0; j < K; ++j) {
            wt[j][i] = W[((size_t)h * D + c0 + i) * K + j];
            pend[j][i] = 0.f;
            gw[j][i] = 0.f;
        }
    cur.seek(r0);
#pragma unroll
    for (int j = 0; j < K - 1; ++j) {
        const long r = r0 - (K - 1) + j;
        if (r >= cur.start && r >= 0) ld<Tin, CPL>(x + ((size_t)r * H + h) * D + c0, win[j]);
        else
#pragma unroll
            for (int i = 0; i < CPL; ++i) win[j][i] = 0.f;
    }
    // rows r0 .. r0 + nr - 1 + K - 1: dy of each row; pend[j] collects dx of
    // row r - (K-1) + j (only rows of r's sequence); row r - (K-1) is complete
    // after row r
    for (int it = 0; it < nr + K - 1; ++it) {
        const long r = r0 + it;
        float dy[CPL];
#pragma unroll
        for (int i = 0; i < CPL; ++i) dy[i] = 0.f;
        long seq_start = -1;
        if (r < rows) {
            cur.advance(r);
            seq_start = cur.start;
            if (r == cur.start)
#pragma unroll
                for (int j = 0; j < K - 1; ++j)
#pragma unroll
                    for (int i = 0; i < CPL; ++i) win[j][i] = 0.f;
            ld<Tin, CPL>(x + ((size_t)r * H + h) * D + c0, win[K - 1]);
            float y[CPL], s[CPL], g[CPL], ss = 0.f, dot = 0.f;
            ld<Tin, CPL>(dout + ((size_t)r * H + h) * D + c0, g);
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < K; ++j) acc = fmaf(wt[j][i], win[j][i], acc);
                y[i] = acc;
                s[i] = acc * sigm(acc);
                ss = fmaf(s[i], s[i], ss);
            }
            float n = 1.f;
            if (l2) {
                n = rsqrtf(warp_sum(ss) + kEps);  // 1 / |s|
#pragma unroll
                for (int i = 0; i < CPL; ++i) dot = fmaf(s[i] * n, g[i], dot);
                dot = warp_sum(dot);
            }
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                const float ds = l2 ? (g[i] - s[i] * n * dot) * n : g[i];
                const float sg = sigm(y[i]);
                dy[i] = ds * sg * (1.f + y[i] * (1.f - sg));
            }
            if (it < nr)  // the filter gradient from this warp's own rows
#pragma unroll
                for (int j = 0; j < K; ++j)
#pragma unroll
                    for (int i = 0; i < CPL; ++i) gw[j][i] = fmaf(dy[i], win[j][i], gw[j][i]);
        }
#pragma unroll
        for (int j = 0; j < K; ++j) {
            const long p = r - (K - 1) + j;
            if (p >= seq_start)
#pragma unroll
                for (int i = 0; i < CPL; ++i) pend[j][i] = fmaf(wt[j][i], dy[i], pend[j][i]);
        }
        const long p0 = r - (K - 1);  // complete now
        if (p0 >= r0 && p0 < r0 + nr) st<Tin, CPL>(dx + ((size_t)p0 * H + h) * D + c0, pend[0]);
#pragma unroll
        for (int j = 0; j < K - 1; ++j)
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                pend[j][i] = pend[j + 1][i];
                win[j][i] = win[j + 1][i];
            }
#pragma unroll
        for (int i = 0; i < CPL; ++i) pend[K - 1][i] = 0.f;
    }
#pragma unroll
    for (int i = 0; i < CPL; ++i)
#pragma unroll
        for (int j = 0; j < K; ++j) dW[c0 + i][j] = gw[j][i];
}

template <typename Tin, int D>
__device__ __forceinline__ void gate_rows_bwd(const Tin *x, const Tin *dout, Tin *dx, bool logsig, long r0, int nr, int h, int H,
                              int lane) {
    constexpr int CPL = D / 32;
    for (int it = 0; it < nr; ++it) {
        const size_t o = ((size_t)(r0 + it) * H + h) * D + lane * CPL;
        float v[CPL], g[CPL];
        ld<Tin, CPL>(x + o, v);
        ld<Tin, CPL>(dout + o, g);
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const float s = sigm(v[i]);
            v[i] = g[i] * (logsig ? 1.f - s : s * (1.f - s));
        }
        st<Tin, CPL>(dx + o, v);
    }
}

template <typename Tin, int DK, int DV, int K>
__global__ void __launch_bounds__(kWarps * 32) prologue_bwd_kernel(PrologueBwdArgs a) {
    constexpr int NC = 2 * DK + DV;  // filter rows of the three paths
    __shared__ float red[kWarps][NC][K];
    const PrologueArgs &f = a.f;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, h = blockIdx.y;
    const long r0 = (long)blockIdx.x * kRowsPerCta + warp * kRowsPerWarp;
    const int nr = r0 < f.rows ? (int)min((long)kRowsPerWarp, f.rows - r0) : 0;
    SeqCursor cur{f.cu, f.N, f.T, 0, 0, 0};
    if (nr > 0) {
        conv_path_bwd<Tin, DK, K>(static_cast<const Tin *>(f.xq), f.Wq, static_cast<const Tin *>(a.dq),
                                  static_cast<Tin *>(a.dxq), true, r0, nr, f.rows, h, f.H, cur, lane, red[warp]);
        conv_path_bwd<Tin, DK, K>(static_cast<const Tin *>(f.xk), f.Wk, static_cast<const Tin *>(a.dk),
                                  static_cast<Tin *>(a.dxk), true, r0, nr, f.rows, h, f.H, cur, lane,
                                  red[warp] + DK);
        conv_path_bwd<Tin, DV, K>(static_cast<const Tin *>(f.xv), f.Wv, static_cast<const Tin *>(a.dv),
                                  static_cast<Tin *>(a.dxv), false, r0, nr, f.rows, h, f.H, cur, lane,
                                  red[warp] + 2 * DK);
        gate_rows_bwd<Tin, DK>(static_cast<const Tin *>(f.xa), static_cast<const Tin *>(a.dla),
                               static_cast<Tin *>(a.dxa), true, r0, nr, h, f.H, lane);
        gate_rows_bwd<Tin, DK>(static_cast<const Tin *>(f.xb), static_cast<const Tin *>(a.db),
                               static_cast<Tin *>(a.dxb), false, r0, nr, h, f.H, lane);
        gate_rows_bwd<Tin, DV>(static_cast<const Tin *>(f.xw), static_cast<const Tin *>(a.dw),
                               static_cast<Tin *>(a.dxw), false, r0, nr, h, f.H, lane);
    } else {
        for (int i = lane; i < NC * K; i += 32) red[warp][i / K][i % K] = 0.f;
    }
    __syncthreads();
    // this CTA's filter-gradient sums, warps added in order
    float *out = a.part + ((size_t)blockIdx.x * f.H + h) * NC * K;
    for (int i = threadIdx.x; i < NC * K; i += blockDim.x) {
        float acc = 0.f;
#pragma unroll
        for (int wi = 0; wi < kWarps; ++wi) acc += red[wi][i / K][i % K];
        out[i] = acc;
    }
}

// dW[h][c][j] = sum over the CTAs (in order) of their sums, split back into
// the three paths' filters.
__global__ void filter_grad_reduce_kernel(const float *part, int nblk, int H, int dk, int dv, int K, float *dWq,
                                          float *dWk, float *dWv) {
    const int NC = 2 * dk + dv;
    const long n = (long)H * NC * K;
    for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
        float acc = 0.f;
        for (int bl = 0; bl < nblk; ++bl) acc += part[(size_t)bl * n + i];
        const int h = (int)(i / ((long)NC * K)), rem = (int)(i % ((long)NC * K)), c = rem / K, j = rem % K;
        if (c < dk) dWq[((size_t)h * dk + c) * K + j] = acc;
        else if (c < 2 * dk) dWk[((size_t)h * dk + c - dk) * K + j] = acc;
        else dWv[((size_t)h * dv + c - 2 * dk) * K + j] = acc;
    }
}

// ---------------------------------------------------------------------------
// Output epilogue: z = o / rms(o) * gamma * silu(g)

struct EpilogueArgs {
    const void *o, *g;
    const float *gamma;  // [D]
    void *z;
    const void *dz;      // backward
    void *dO, *dg;
    float *part;         // backward: per CTA dgamma sums [grid.x * H][D]
    long rows;
    int H;
};

template <typename Tin, int D>
__global__ void __launch_bounds__(kWarps * 32) epilogue_fwd_kernel(EpilogueArgs a) {
    constexpr int CPL = D / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, h = blockIdx.y;
    const long r0 = (long)blockIdx.x * kRowsPerCta + warp * kRowsPerWarp;
    float gm[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) gm[i] = a.gamma[lane * CPL + i];
    for (int it = 0; it < kRowsPerWarp && r0 + it < a.rows; ++it) {
        const size_t off = ((size_t)(r0 + it) * a.H + h) * D + lane * CPL;
        float o[CPL], g[CPL], ss = 0.f;
        ld<Tin, CPL>(static_cast<const Tin *>(a.o) + off, o);
        ld<Tin, CPL>(static_cast<const Tin *>(a.g) + off, g);
#pragma unroll
        for (int i = 0; i < CPL; ++i) ss = fmaf(o[i], o[i], ss);
        const float r = rsqrtf(warp_sum(ss) / D + kEps);
#pragma unroll
        for (int i = 0; i < CPL; ++i) o[i] = o[i] * r * gm[i] * g[i] * sigm(g[i]);
        st<Tin, CPL>(static_cast<Tin *>(a.z) + off, o);
    }
}

template <typename Tin, int D>
__global__ void __launch_bounds__(kWarps * 32) epilogue_bwd_kernel(EpilogueArgs a) {
    constexpr int CPL = D / 32;
    __shared__ float red[kWarps][D];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, h = blockIdx.y;
    const long r0 = (long)blockIdx.x * kRowsPerCta + warp * kRowsPerWarp;
    float gm[CPL], dgm[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        gm[i] = a.gamma[lane * CPL + i];
        dgm[i] = 0.f;
    }
    for (int it = 0; it < kRowsPerWarp && r0 + it < a.rows; ++it) {
        const size_t off = ((size_t)(r0 + it) * a.H + h) * D + lane * CPL;
        float o[CPL], g[CPL], dz[CPL], ss = 0.f;
        ld<Tin, CPL>(static_cast<const Tin *>(a.o) + off, o);
        ld<Tin, CPL>(static_cast<const Tin *>(a.g) + off, g);
        ld<Tin, CPL>(static_cast<const Tin *>(a.dz) + off, dz);
#pragma unroll
        for (int i = 0; i < CPL; ++i) ss = fmaf(o[i], o[i], ss);
        const float r = rsqrtf(warp_sum(ss) / D + kEps);
        float dn[CPL], m = 0.f, dgo[CPL];
#pragma unroll
        for (int i = 0; i < CPL; ++i) {
            const float sg = sigm(g[i]), n = o[i] * r, sl = g[i] * sg;
            dn[i] = dz[i] * gm[i] * sl;
            m = fmaf(n, dn[i], m);
            dgm[i] = fmaf(dz[i] * n, sl, dgm[i]);
            dgo[i] = dz[i] * n * gm[i] * sg * (1.f + g[i] * (1.f - sg));
        }
        m = warp_sum(m) / D;
#pragma unroll
        for (int i = 0; i < CPL; ++i) o[i] = r * (dn[i] - o[i] * r * m);
        st<Tin, CPL>(static_cast<Tin *>(a.dO) + off, o);
        st<Tin, CPL>(static_cast<Tin *>(a.dg) + off, dgo);
    }
#pragma unroll
    for (int i = 0; i < CPL; ++i) red[warp][lane * CPL + i] = dgm[i];
    __syncthreads();
    float *out = a.part + ((size_t)blockIdx.x * a.H + h) * D;
    for (int i = threadIdx.x; i < D; i += blockDim.x) {
        float acc = 0.f;
#pragma unroll
        for (int wi = 0; wi < kWarps; ++wi) acc += red[wi][i];
        out[i] = acc;
    }
}

__global__ void gamma_grad_reduce_kernel(const float *part, int nblk, int D, float *dgamma) {
    for (int j = threadIdx.x; j < D; j += blockDim.x) {
        float acc = 0.f;
        for (int bl = 0; bl < nblk; ++bl) acc += part[(size_t)bl * D + j];
        dgamma[j] = acc;
    }
}

unsigned row_blocks(long rows) { return (unsigned)((rows + kRowsPerCta - 1) / kRowsPerCta); }

template <typename Tin, int DK, int DV>
cudaError_t launch_prologue_k(const PrologueArgs &a, const PrologueBwdArgs *b, cudaStream_t s) {
    const dim3 grid(row_blocks(a.rows), (unsigned)a.H), block(kWarps * 32);
    switch (a.K) {
#define GDN2_K(KK)                                                              \
    case KK:                                                                    \
        if (b) prologue_bwd_kernel<Tin, DK, DV, KK><<<grid, block, 0, s>>>(*b); \
        else prologue_fwd_kernel<Tin, DK, DV, KK><<<grid, block, 0, s>>>(a);    \
        break;
        GDN2_K(1) GDN2_K(2) GDN2_K(3) GDN2_K(4)
#undef GDN2_K
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_prologue_t(const PrologueArgs &a, const PrologueBwdArgs *b, int dk, int dv, cudaStream_t s) {
    if (dk == 128 && dv == 128) return launch_prologue_k<Tin, 128, 128>(a, b, s);
    if (dk == 128 && dv == 64) return launch_prologue_k<Tin, 128, 64>(a, b, s);
    if (dk == 64 && dv == 128) return launch_prologue_k<Tin, 64, 128>(a, b, s);
    return launch_prologue_k<Tin, 64, 64>(a, b, s);
}

int launch_status(cudaError_t e) {
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return GDN2_ERR_CUDA;
    }
    return GDN2_OK;
}

bool a16(const void *p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_dims(int dk, int dv) { return (dk == 64 || dk == 128) && (dv == 64 || dv == 128); }

}  // namespace layer
}  // namespace gdn2

using namespace gdn2::layer;

extern "C" {

int gdn2_prologue_fwd(const void *xq, const void *xk, const void *xv, const float *Wq, const float *Wk,
                      const float *Wv, int K, const void *xa, const void *xb, const void *xw, void *q, void *k,
                      void *v, void *log_alpha, void *b, void *w, const int *cu_seqlens, int B, int T, int H, int dk,
                      int dv, int dtype, cudaStream_t stream) {
    if (B < 0 || T < 0 || H < 0) return GDN2_ERR_INVALID_ARG;
    if (!ok_dims(dk, dv) || (dtype != GDN2_BF16 && dtype != GDN2_FP32) || K < 1 || K > kMaxConv)
        return GDN2_ERR_UNSUPPORTED;
    const long rows = cu_seqlens ? (long)T : (long)B * T;  // packed: B sequences in T rows
    if (rows == 0 || H == 0 || B == 0) return GDN2_OK;
    const void *ptrs[] = {xq, xk, xv, Wq, Wk, Wv, xa, xb, xw, q, k, v, log_alpha, b, w};
    for (const void *p : ptrs)
        if (!a16(p)) return GDN2_ERR_INVALID_ARG;
    if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return GDN2_ERR_INVALID_ARG;
    PrologueArgs a{xq, xk, xv, xa, xb, xw, Wq, Wk, Wv, q, k, v, log_alpha, b, w, rows, H, K, T, cu_seqlens, B};
    return launch_status(dtype == GDN2_BF16 ? launch_prologue_t<__nv_bfloat16>(a, nullptr, dk, dv, stream)
                                            : launch_prologue_t<float>(a, nullptr, dk, dv, stream));
}

size_t gdn2_prologue_bwd_workspace(int B, int T, int H, int dk, int dv, int K, int packed) {
    if (B <= 0 || T <= 0 || H <= 0 || !ok_dims(dk, dv) || K < 1 || K > kMaxConv) return 0;
    const long rows = packed ? (long)T : (long)B * T;
    return (size_t)row_blocks(rows) * H * (2 * dk + dv) * K * sizeof(float);
}

int gdn2_prologue_bwd(const void *xq, const void *xk, const void *xv, const float *Wq, const float *Wk,
                      const float *Wv, int K, const void *xa, const void *xb, const void *xw, const void *dq,
                      const void *dk_, const void *dv_, const void *dlog_alpha, const void *db, const void *dw,
                      void *dxq, void *dxk, void *dxv, float *dWq, float *dWk, float *dWv, void *dxa, void *dxb,
                      void *dxw, const int *cu_seqlens, int B, int T, int H, int dk, int dv, int dtype, void *ws,
                      size_t ws_bytes, cudaStream_t stream) {
    if (B < 0 || T < 0 || H < 0) return GDN2_ERR_INVALID_ARG;
    if (!ok_dims(dk, dv) || (dtype != GDN2_BF16 && dtype != GDN2_FP32) || K < 1 || K > kMaxConv)
        return GDN2_ERR_UNSUPPORTED;
    const long rows = cu_seqlens ? (long)T : (long)B * T;
    if (rows == 0 || H == 0 || B == 0) return GDN2_OK;  // (the filter gradients are not written)
    const void *ptrs[] = {xq, xk, xv, Wq, Wk, Wv, xa, xb, xw, dq, dk_, dv_, dlog_alpha, db, dw,
                          dxq, dxk, dxv, dWq, dWk, dWv, dxa, dxb, dxw};
    for (const void *p : ptrs)
        if (!a16(p)) return GDN2_ERR_INVALID_ARG;
    if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return GDN2_ERR_INVALID_ARG;
    const size_t need = gdn2_prologue_bwd_workspace(B, T, H, dk, dv, K, cu_seqlens != nullptr);
    if (ws_bytes < need || !a16(ws)) return GDN2_ERR_WORKSPACE;
    PrologueBwdArgs a{{xq, xk, xv, xa, xb, xw, Wq, Wk, Wv, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                       rows, H, K, T, cu_seqlens, B},
                      dq, dk_, dv_, dlog_alpha, db, dw, dxq, dxk, dxv, dxa, dxb, dxw, static_cast<float *>(ws)};
    cudaError_t e = dtype == GDN2_BF16 ? launch_prologue_t<__nv_bfloat16>(a.f, &a, dk, dv, stream)
                                       : launch_prologue_t<float>(a.f, &a, dk, dv, stream);
    if (e != cudaSuccess) return launch_status(e);
    const long n = (long)H * (2 * dk + dv) * K;
    filter_grad_reduce_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(
        a.part, (int)row_blocks(rows), H, dk, dv, K, dWq, dWk, dWv);
    return launch_status(cudaGetLastError());
}

int gdn2_output_gate_fwd(const void *o, const void *g, const float *gamma, void *z, long long rows, int H, int dv,
                         int dtype, cudaStream_t stream) {
    if (rows < 0 || H < 0) return GDN2_ERR_INVALID_ARG;
    if ((dv != 64 && dv != 128) || (dtype != GDN2_BF16 && dtype != GDN2_FP32)) return GDN2_ERR_UNSUPPORTED;
    if (rows == 0 || H == 0) return GDN2_OK;
    if (!a16(o) || !a16(g) || !a16(gamma) || !a16(z)) return GDN2_ERR_INVALID_ARG;
    EpilogueArgs a{o, g, gamma, z, nullptr, nullptr, nullptr, nullptr, (long)rows, H};
    const dim3 grid(row_blocks(rows), (unsigned)H), block(kWarps * 32);
    if (dtype == GDN2_BF16) {
        if (dv == 128) epilogue_fwd_kernel<__nv_bfloat16, 128><<<grid, block, 0, stream>>>(a);
        else epilogue_fwd_kernel<__nv_bfloat16, 64><<<grid, block, 0, stream>>>(a);
    } else {
        if (dv == 128) epilogue_fwd_kernel<float, 128><<<grid, block, 0, stream>>>(a);
        else epilogue_fwd_kernel<float, 64><<<grid, block, 0, stream>>>(a);
    }
    return launch_status(cudaGetLastError());
}

size_t gdn2_output_gate_bwd_workspace(long long rows, int H, int dv) {
    if (rows <= 0 || H <= 0 || (dv != 64 && dv != 128)) return 0;
    return (size_t)row_blocks(rows) * H * dv * sizeof(float);
}

int gdn2_output_gate_bwd(const void *o, const void *g, const float *gamma, const void *dz, void *dO, void *dg,
                         float *dgamma, long long rows, int H, int dv, int dtype, void *ws, size_t ws_bytes,
                         cudaStream_t stream) {
    if (rows < 0 || H < 0) return GDN2_ERR_INVALID_ARG;
    if ((dv != 64 && dv != 128) || (dtype != GDN2_BF16 && dtype != GDN2_FP32)) return GDN2_ERR_UNSUPPORTED;
    if (rows == 0 || H == 0) return GDN2_OK;
    if (!a16(o) || !a16(g) || !a16(gamma) || !a16(dz) || !a16(dO) || !a16(dg) || !a16(dgamma))
        return GDN2_ERR_INVALID_ARG;
    if (ws_bytes < gdn2_output_gate_bwd_workspace(rows, H, dv) || !a16(ws)) return GDN2_ERR_WORKSPACE;
    EpilogueArgs a{o, g, gamma, nullptr, dz, dO, dg, static_cast<float *>(ws), (long)rows, H};
    const dim3 grid(row_blocks(rows), (unsigned)H), block(kWarps * 32);
    if (dtype == GDN2_BF16) {
        if (dv == 128) epilogue_bwd_kernel<__nv_bfloat16, 128><<<grid, block, 0, stream>>>(a);
        else epilogue_bwd_kernel<__nv_bfloat16, 64><<<grid, block, 0, stream>>>(a);
    } else {
        if (dv == 128) epilogue_bwd_kernel<float, 128><<<grid, block, 0, stream>>>(a);
        else epilogue_bwd_kernel<float, 64><<<grid, block, 0, stream>>>(a);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return launch_status(e);
    gamma_grad_reduce_kernel<<<1, 128, 0, stream>>>(a.part, (int)(row_blocks(rows) * H), dv, dgamma);
    return launch_status(cudaGetLastError());
}

}  // extern "C"
