// Token-recurrent kernels: the decode step and the fp32 precision mode.
//
// One CTA of 256 threads owns one (batch, head) state S [DK x DV] (fp32) and
// holds it in registers: a warp covers whole rows with 128-bit column groups
// (lane -> 4 consecutive value columns), so every state row is one coalesced
// 512-byte (DV = 128) or 256-byte (DV = 64) access.  Per token
//
//     S' = Diag(alpha) S,   u = w.v - S'^T (b.k),   S = S' + k u^T,
//     o  = S^T q = S'^T q + (q.k) u
//
// ("Why NVIDIA Gated DeltaNet-2 separates erase and write gates", section
// "Gated Delta Rule-2: per-channel erase/write split", recurrence).  The two
// reductions over the key axis (S'^T (b.k) and S'^T q) are taken in one pass
// over the registers (per-thread partial sums, a warp shuffle when two rows
// share a warp, then a cross-warp sum through shared memory), so the state is
// read from HBM once and written once.
//
// The backward kernel is the reverse-time adjoint of the same four lines (the
// gate-aware vector-Jacobian product of that section), replaying each
// 64-token segment from an fp32 checkpoint.
#include "common.cuh"
#include "launch.h"

namespace gdn2 {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <int DK, int DV>
struct Layout {
    static constexpr int LPR = DV / 4;                 // lanes per state row
    static constexpr int RPW = 32 / LPR;               // rows per warp per pass
    static constexpr int RT = DK / (kWarps * RPW);     // rows held per thread
    static_assert(RT >= 1 && DK % (kWarps * RPW) == 0, "state layout");
    __device__ static int row(int i, int warp, int lane) { return (i * kWarps + warp) * RPW + lane / LPR; }
    __device__ static int cg(int lane) { return lane % LPR; }
};

// Sum over the LPR lanes that share one state row.
template <int LPR>
__device__ __forceinline__ float row_sum(float x) {
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Element offset of token t of a sequence whose tokens are the rows row0 .. of
// a token tensor [rows][H][D] (head h).
__device__ __forceinline__ size_t tok_off(size_t row0, int t, int H, int h, int D) {
    return ((row0 + t) * H + h) * (size_t)D;
}

// Loads one token's gates into shared memory.  Key side: alpha, (b.k).alpha,
// q.alpha, k, b.k; value side: w.v, v, w.  Returns q.k in *qk (valid after the
// caller's next __syncthreads through s_qkp).
template <typename Tin, int DK, int DV>
__device__ __forceinline__ void load_token(const RecurrentArgs &a, size_t row0, int t, int h,
                                           float *s_a, float *s_ga, float *s_qa, float *s_k,
                                           float *s_g, float *s_wv, float *s_v, float *s_w,
                                           float *s_qkp) {
    const int tid = threadIdx.x;
    // a scalar gate (KDA: beta for b and w; GDN: also the decay) is one
    // element per token and head
    const size_t os = (row0 + t) * a.H + h;
    if (tid < DK) {
        const size_t o = tok_off(row0, t, a.H, h, DK);
        const float q = to_f32(static_cast<const Tin *>(a.q)[o + tid]);
        const float k = to_f32(static_cast<const Tin *>(a.k)[o + tid]);
        const float la = to_f32(static_cast<const Tin *>(a.log_alpha)[a.gates == kGatesGDN ? os : o + tid]);
        const float bg = to_f32(static_cast<const Tin *>(a.b)[a.gates == kGatesFull ? o + tid : os]);
        const float al = expf(la);
        const float g = bg * k;
        s_a[tid] = al;
        s_ga[tid] = g * al;
        s_qa[tid] = q * al;
        s_k[tid] = k;
        if (s_g) s_g[tid] = g;
        const float qk = warp_sum(q * k);
        if ((tid & 31) == 0) s_qkp[tid >> 5] = qk;
    } else if (tid < DK + DV) {
        const int j = tid - DK;
        const size_t o = tok_off(row0, t, a.H, h, DV);
        const float v = to_f32(static_cast<const Tin *>(a.v)[o + j]);
        const float w = to_f32(static_cast<const Tin *>(a.w)[a.gates == kGatesFull ? o + j : os]);
        s_wv[j] = w * v;
        if (s_v) s_v[j] = v;
        if (s_w) s_w[j] = w;
    }
}

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kThreads) recurrent_fwd_kernel(RecurrentArgs a) {
    using L = Layout<DK, DV>;
    const int bh = blockIdx.x;
    const int b = bh / a.H, h = bh % a.H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, cg = L::cg(lane);
    const SeqView sv = seq_view(a.cu_seqlens, b, h, a.B, a.T, a.H);
    if (!sv.ok) return;  // packed-sequence offsets out of range

    __shared__ float s_a[DK], s_ga[DK], s_qa[DK], s_k[DK], s_wv[DV], s_u[DV];
    __shared__ float s_red[2][kWarps][DV];
    __shared__ float s_qkp[kWarps];

    const size_t sbase = (size_t)bh * DK * DV;
    float4 S[L::RT];
#pragma unroll
    for (int i = 0; i < L::RT; ++i) {
        const int row = L::row(i, warp, lane);
        S[i] = a.S_in ? ld_stream(reinterpret_cast<const float4 *>(a.S_in + sbase + (size_t)row * DV) + cg)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }

    for (int t = 0; t < sv.len; ++t) {
        load_token<Tin, DK, DV>(a, sv.row0, t, h, s_a, s_ga, s_qa, s_k, nullptr, s_wv, nullptr, nullptr, s_qkp);
        __syncthreads();
        float4 p = make_float4(0.f, 0.f, 0.f, 0.f), r = p;
#pragma unroll
        for (int i = 0; i < L::RT; ++i) {
            const int row = L::row(i, warp, lane);
            const float ga = s_ga[row], qa = s_qa[row];
            p.x += ga * S[i].x; p.y += ga * S[i].y; p.z += ga * S[i].z; p.w += ga * S[i].w;
            r.x += qa * S[i].x; r.y += qa * S[i].y; r.z += qa * S[i].z; r.w += qa * S[i].w;
        }
        if (L::RPW == 2) {
            p.x += __shfl_xor_sync(0xffffffffu, p.x, 16); p.y += __shfl_xor_sync(0xffffffffu, p.y, 16);
            p.z += __shfl_xor_sync(0xffffffffu, p.z, 16); p.w += __shfl_xor_sync(0xffffffffu, p.w, 16);
            r.x += __shfl_xor_sync(0xffffffffu, r.x, 16); r.y += __shfl_xor_sync(0xffffffffu, r.y, 16);
            r.z += __shfl_xor_sync(0xffffffffu, r.z, 16); r.w += __shfl_xor_sync(0xffffffffu, r.w, 16);
        }
        if (lane < L::LPR) {
            *reinterpret_cast<float4 *>(&s_red[0][warp][4 * cg]) = p;
            *reinterpret_cast<float4 *>(&s_red[1][warp][4 * cg]) = r;
        }
        __syncthreads();
        if (threadIdx.x < DV) {
            const int j = threadIdx.x;
            float pj = 0.f, rj = 0.f, qk = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) { pj += s_red[0][w][j]; rj += s_red[1][w][j]; }
#pragma unroll
            for (int w = 0; w < DK / 32; ++w) qk += s_qkp[w];
            const float u = s_wv[j] - pj;
            s_u[j] = u;
            static_cast<Tin *>(a.o)[tok_off(sv.row0, t, a.H, h, DV) + j] = from_f32<Tin>(rj + qk * u);
        }
        __syncthreads();
        const float4 u4 = *reinterpret_cast<const float4 *>(&s_u[4 * cg]);
#pragma unroll
        for (int i = 0; i < L::RT; ++i) {
            const int row = L::row(i, warp, lane);
            const float al = s_a[row], k = s_k[row];
            S[i].x = al * S[i].x + k * u4.x; S[i].y = al * S[i].y + k * u4.y;
            S[i].z = al * S[i].z + k * u4.z; S[i].w = al * S[i].w + k * u4.w;
        }
        __syncthreads();
    }
    if (a.S_out) {
#pragma unroll
        for (int i = 0; i < L::RT; ++i) {
            const int row = L::row(i, warp, lane);
            st_stream(reinterpret_cast<float4 *>(a.S_out + sbase + (size_t)row * DV) + cg, S[i]);
        }
    }
}

// ---------------------------------------------------------------------------
// Reverse-time backward (fp32 precision mode).
//
// Workspace: the checkpoints [DK x DV] at every 64-token segment start, one
// slot per segment as the chunk path lays out its per-chunk tiles (SeqView),
// then per (b,h) one 64-token segment of decayed states S'_t [64][DK x DV]
// and edits u_t [64][DV].

constexpr int kSeg = 64;
static_assert(kSeg == 64, "checkpoint slots follow the 64-token chunk slots");

template <int DK, int DV>
__host__ __device__ constexpr size_t bwd_seg_floats() {
    return (size_t)kSeg * DK * DV + (size_t)kSeg * DV;
}

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kThreads) recurrent_bwd_kernel(RecurrentBwdArgs a) {
    using L = Layout<DK, DV>;
    const int bh = blockIdx.x;
    const int b = bh / a.H, h = bh % a.H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, cg = L::cg(lane);
    const SeqView sv = seq_view(a.cu_seqlens, b, h, a.B, a.T, a.H);
    if (!sv.ok) return;  // packed-sequence offsets out of range
    const int T = sv.len, nseg = sv.nchunks;

    __shared__ float s_a[DK], s_ga[DK], s_qa[DK], s_k[DK], s_g[DK], s_q[DK], s_b[DK];
    __shared__ float s_wv[DV], s_v[DV], s_w[DV], s_u[DV], s_do[DV], s_du[DV];
    __shared__ float s_red[kWarps][DV];
    __shared__ float s_qkp[kWarps];
    __shared__ float s_udo;

    const size_t nslots = chunk_slots(a.B, a.T, a.H, a.cu_seqlens != nullptr);
    float *ckpt = a.ws + sv.cslot * DK * DV;
    float *segSp = a.ws + nslots * DK * DV + (size_t)bh * bwd_seg_floats<DK, DV>();
    float *segU = segSp + (size_t)kSeg * DK * DV;
    const size_t sbase = (size_t)bh * DK * DV;
    RecurrentArgs fa{a.q, a.k, a.v, a.log_alpha, a.b, a.w, nullptr, nullptr, nullptr, a.B, a.T, a.H, a.cu_seqlens};

    // 1. forward pass, checkpoint at every segment start
    float4 S[L::RT];
#pragma unroll
    for (int i = 0; i < L::RT; ++i) {
        const int row = L::row(i, warp, lane);
        S[i] = a.S0 ? reinterpret_cast<const float4 *>(a.S0 + sbase + (size_t)row * DV)[cg]
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int t = 0; t < T; ++t) {
        if (t % kSeg == 0) {
#pragma unroll
            for (int i = 0; i < L::RT; ++i) {
                const int row = L::row(i, warp, lane);
                reinterpret_cast<float4 *>(ckpt + (size_t)(t / kSeg) * DK * DV + (size_t)row * DV)[cg] = S[i];
            }
        }
        load_token<Tin, DK, DV>(fa, sv.row0, t, h, s_a, s_ga, s_qa, s_k, nullptr, s_wv, nullptr, nullptr, s_qkp);
        __syncthreads();
        float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < L::RT; ++i) {
            const float ga = s_ga[L::row(i, warp, lane)];
            p.x += ga * S[i].x; p.y += ga * S[i].y; p.z += ga * S[i].z; p.w += ga * S[i].w;
        }
        if (L::RPW == 2) {
            p.x += __shfl_xor_sync(0xffffffffu, p.x, 16); p.y += __shfl_xor_sync(0xffffffffu, p.y, 16);
            p.z += __shfl_xor_sync(0xffffffffu, p.z, 16); p.w += __shfl_xor_sync(0xffffffffu, p.w, 16);
        }
        if (lane < L::LPR) *reinterpret_cast<float4 *>(&s_red[warp][4 * cg]) = p;
        __syncthreads();
        if (threadIdx.x < DV) {
            float pj = 0.f;
            for (int w = 0; w < kWarps; ++w) pj += s_red[w][threadIdx.x];
            s_u[threadIdx.x] = s_wv[threadIdx.x] - pj;
        }
        __syncthreads();
        const float4 u4 = *reinterpret_cast<const float4 *>(&s_u[4 * cg]);
#pragma unroll
        for (int i = 0; i < L::RT; ++i) {
            const int row = L::row(i, warp, lane);
            const float al = s_a[row], k = s_k[row];
            S[i].x = al * S[i].x + k * u4.x; S[i].y = al * S[i].y + k * u4.y;
            S[i].z = al * S[i].z + k * u4.z; S[i].w = al * S[i].w + k * u4.w;
        }
        __syncthreads();
    }

    // 2. adjoint state Shat = dL/dS_T
    float4 Sh[L::RT];
#pragma unroll
    for (int i = 0; i < L::RT; ++i) {
        const int row = L::row(i, warp, lane);
        Sh[i] = a.dS_T ? reinterpret_cast<const float4 *>(a.dS_T + sbase + (size_t)row * DV)[cg]
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    }

    for (int seg = nseg - 1; seg >= 0; --seg) {
        const int t0 = seg * kSeg, t1 = min(T, t0 + kSeg);
        // 2a. replay the segment: S'_t and u_t into the workspace
#pragma unroll
        for (int i = 0; i < L::RT; ++i) {
            const int row = L::row(i, warp, lane);
            S[i] = reinterpret_cast<const float4 *>(ckpt + (size_t)seg * DK * DV + (size_t)row * DV)[cg];
        }
        for (int t = t0; t < t1; ++t) {
            load_token<Tin, DK, DV>(fa, sv.row0, t, h, s_a, s_ga, s_qa, s_k, nullptr, s_wv, nullptr, nullptr, s_qkp);
            __syncthreads();
            float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
            float *Sp = segSp + (size_t)(t - t0) * DK * DV;
#pragma unroll
            for (int i = 0; i < L::RT; ++i) {
                const int row = L::row(i, warp, lane);
                const float al = s_a[row], ga = s_ga[row];
                const float4 sp = make_float4(al * S[i].x, al * S[i].y, al * S[i].z, al * S[i].w);
                reinterpret_cast<float4 *>(Sp + (size_t)row * DV)[cg] = sp;
                p.x += ga * S[i].x; p.y += ga * S[i].y; p.z += ga * S[i].z; p.w += ga * S[i].w;
                S[i] = sp;
            }
            if (L::RPW == 2) {
                p.x += __shfl_xor_sync(0xffffffffu, p.x, 16); p.y += __shfl_xor_sync(0xffffffffu, p.y, 16);
                p.z += __shfl_xor_sync(0xffffffffu, p.z, 16); p.w += __shfl_xor_sync(0xffffffffu, p.w, 16);
            }
            if (lane < L::LPR) *reinterpret_cast<float4 *>(&s_red[warp][4 * cg]) = p;
            __syncthreads();
            if (threadIdx.x < DV) {
                float pj = 0.f;
                for (int w = 0; w < kWarps; ++w) pj += s_red[w][threadIdx.x];
                const float u = s_wv[threadIdx.x] - pj;
                s_u[threadIdx.x] = u;
                segU[(size_t)(t - t0) * DV + threadIdx.x] = u;
            }
            __syncthreads();
            const float4 u4 = *reinterpret_cast<const float4 *>(&s_u[4 * cg]);
#pragma unroll
            for (int i = 0; i < L::RT; ++i) {
                const float k = s_k[L::row(i, warp, lane)];
                S[i].x += k * u4.x; S[i].y += k * u4.y; S[i].z += k * u4.z; S[i].w += k * u4.w;
            }
            __syncthreads();
        }
        // 2b. reverse over the segment
        for (int t = t1 - 1; t >= t0; --t) {
            const int tid = threadIdx.x;
            if (tid < DK) {
                const size_t o = tok_off(sv.row0, t, a.H, h, DK);
                const float q = to_f32(static_cast<const Tin *>(a.q)[o + tid]);
                const float k = to_f32(static_cast<const Tin *>(a.k)[o + tid]);
                const float la = to_f32(static_cast<const Tin *>(a.log_alpha)[o + tid]);
                const float bg = to_f32(static_cast<const Tin *>(a.b)[o + tid]);
                s_q[tid] = q; s_k[tid] = k; s_b[tid] = bg; s_g[tid] = bg * k; s_a[tid] = expf(la);
            } else if (tid < DK + DV) {
                const int j = tid - DK;
                const size_t o = tok_off(sv.row0, t, a.H, h, DV);
                s_v[j] = to_f32(static_cast<const Tin *>(a.v)[o + j]);
                s_w[j] = to_f32(static_cast<const Tin *>(a.w)[o + j]);
                s_do[j] = to_f32(static_cast<const Tin *>(a.dO)[o + j]);
                s_u[j] = segU[(size_t)(t - t0) * DV + j];
            }
            __syncthreads();
            if (warp == 0) {
                float x = 0.f;
                for (int j = lane; j < DV; j += 32) x += s_u[j] * s_do[j];
                x = warp_sum(x);
                if (lane == 0) s_udo = x;
            }
            const float *Sp = segSp + (size_t)(t - t0) * DK * DV;
            float4 sp[L::RT];
            const float4 do4 = *reinterpret_cast<const float4 *>(&s_do[4 * cg]);
            const float4 u4 = *reinterpret_cast<const float4 *>(&s_u[4 * cg]);
            float dq_p[L::RT], dk_p[L::RT];
            float4 cdu = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int i = 0; i < L::RT; ++i) {
                const int row = L::row(i, warp, lane);
                sp[i] = reinterpret_cast<const float4 *>(Sp + (size_t)row * DV)[cg];
                const float q = s_q[row], k = s_k[row];
                // Shat += q do^T
                Sh[i].x += q * do4.x; Sh[i].y += q * do4.y; Sh[i].z += q * do4.z; Sh[i].w += q * do4.w;
                // dq = S'_t do (+ k (u.do), added after the row sum)
                dq_p[i] = sp[i].x * do4.x + sp[i].y * do4.y + sp[i].z * do4.z + sp[i].w * do4.w;
                // dk = Shat u
                dk_p[i] = Sh[i].x * u4.x + Sh[i].y * u4.y + Sh[i].z * u4.z + Sh[i].w * u4.w;
                // du = Shat^T k
                cdu.x += k * Sh[i].x; cdu.y += k * Sh[i].y; cdu.z += k * Sh[i].z; cdu.w += k * Sh[i].w;
            }
            if (L::RPW == 2) {
                cdu.x += __shfl_xor_sync(0xffffffffu, cdu.x, 16); cdu.y += __shfl_xor_sync(0xffffffffu, cdu.y, 16);
                cdu.z += __shfl_xor_sync(0xffffffffu, cdu.z, 16); cdu.w += __shfl_xor_sync(0xffffffffu, cdu.w, 16);
            }
            if (lane < L::LPR) *reinterpret_cast<float4 *>(&s_red[warp][4 * cg]) = cdu;
            __syncthreads();
            if (tid < DV) {
                float x = 0.f;
                for (int w = 0; w < kWarps; ++w) x += s_red[w][tid];
                s_du[tid] = x;
                const size_t o = tok_off(sv.row0, t, a.H, h, DV);
                static_cast<Tin *>(a.dw)[o + tid] = from_f32<Tin>(x * s_v[tid]);
                static_cast<Tin *>(a.dv)[o + tid] = from_f32<Tin>(x * s_w[tid]);
            }
            __syncthreads();
            const float4 du4 = *reinterpret_cast<const float4 *>(&s_du[4 * cg]);
            const float udo = s_udo;
            const size_t ok = tok_off(sv.row0, t, a.H, h, DK);
#pragma unroll
            for (int i = 0; i < L::RT; ++i) {
                const int row = L::row(i, warp, lane);
                const float g = s_g[row], al = s_a[row];
                float dg = -(sp[i].x * du4.x + sp[i].y * du4.y + sp[i].z * du4.z + sp[i].w * du4.w);
                float4 d;
                d.x = Sh[i].x - g * du4.x; d.y = Sh[i].y - g * du4.y;
                d.z = Sh[i].z - g * du4.z; d.w = Sh[i].w - g * du4.w;
                float dla = d.x * sp[i].x + d.y * sp[i].y + d.z * sp[i].z + d.w * sp[i].w;
                Sh[i].x = al * d.x; Sh[i].y = al * d.y; Sh[i].z = al * d.z; Sh[i].w = al * d.w;
                const float dq = row_sum<L::LPR>(dq_p[i]);
                const float dk = row_sum<L::LPR>(dk_p[i]);
                dg = row_sum<L::LPR>(dg);
                dla = row_sum<L::LPR>(dla);
                if (cg == 0) {
                    const float k = s_k[row];
                    static_cast<Tin *>(a.dq)[ok + row] = from_f32<Tin>(dq + k * udo);
                    static_cast<Tin *>(a.dk)[ok + row] = from_f32<Tin>(dk + dg * s_b[row]);
                    static_cast<Tin *>(a.db)[ok + row] = from_f32<Tin>(dg * k);
                    static_cast<Tin *>(a.dlog_alpha)[ok + row] = from_f32<Tin>(dla);
                }
            }
            __syncthreads();
        }
    }
    if (a.dS0) {
#pragma unroll
        for (int i = 0; i < L::RT; ++i) {
            const int row = L::row(i, warp, lane);
            reinterpret_cast<float4 *>(a.dS0 + sbase + (size_t)row * DV)[cg] = Sh[i];
        }
    }
}

template <typename Tin, int DK, int DV>
cudaError_t launch_fwd_t(const RecurrentArgs &a, cudaStream_t s) {
    recurrent_fwd_kernel<Tin, DK, DV><<<(unsigned)(a.B * a.H), kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

template <typename Tin, int DK, int DV>
cudaError_t launch_bwd_t(const RecurrentBwdArgs &a, cudaStream_t s) {
    recurrent_bwd_kernel<Tin, DK, DV><<<(unsigned)(a.B * a.H), kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t dispatch_fwd(const RecurrentArgs &a, int dk, int dv, cudaStream_t s) {
    if (dk == 128 && dv == 128) return launch_fwd_t<Tin, 128, 128>(a, s);
    if (dk == 128 && dv == 64) return launch_fwd_t<Tin, 128, 64>(a, s);
    if (dk == 64 && dv == 128) return launch_fwd_t<Tin, 64, 128>(a, s);
    return launch_fwd_t<Tin, 64, 64>(a, s);
}

template <typename Tin>
cudaError_t dispatch_bwd(const RecurrentBwdArgs &a, int dk, int dv, cudaStream_t s) {
    if (dk == 128 && dv == 128) return launch_bwd_t<Tin, 128, 128>(a, s);
    if (dk == 128 && dv == 64) return launch_bwd_t<Tin, 128, 64>(a, s);
    if (dk == 64 && dv == 128) return launch_bwd_t<Tin, 64, 128>(a, s);
    return launch_bwd_t<Tin, 64, 64>(a, s);
}

}  // namespace

cudaError_t launch_recurrent_fwd(const RecurrentArgs &a, int dk, int dv, bool bf16, cudaStream_t s) {
    return bf16 ? dispatch_fwd<__nv_bfloat16>(a, dk, dv, s) : dispatch_fwd<float>(a, dk, dv, s);
}

cudaError_t launch_recurrent_bwd(const RecurrentBwdArgs &a, int dk, int dv, bool bf16, cudaStream_t s) {
    return bf16 ? dispatch_bwd<__nv_bfloat16>(a, dk, dv, s) : dispatch_bwd<float>(a, dk, dv, s);
}

size_t recurrent_bwd_ws_bytes(int B, int T, int H, int dk, int dv, bool varlen) {
    return 4 * (chunk_slots(B, T, H, varlen) * dk * dv + (size_t)B * H * ((size_t)kSeg * dk * dv + (size_t)kSeg * dv));
}

}  // namespace gdn2
