// Chunk-parallel forward of the GDN-2 mixer on the tensor cores (bf16 in,
// fp32 accumulate, fp32 state).
//
// Method: "Why NVIDIA Gated DeltaNet-2 separates erase and write gates"
// (axbrief), section "Gated Delta Rule-2: per-channel erase/write split": the
// recurrence S_t = (I - k_t (b_t . k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t . v_t)^T,
// chunks of C = 64 tokens, and the WY form that turns a chunk of rank-1 edits
// into one triangular solve plus matrix products (laonpeople Gated DeltaNet
// page, section on parallel computation / WY representation).
//
// One CTA (8 warps) owns one (batch, head) sequence and walks its chunks in
// order.  For a chunk with start state S (L = in-chunk cumulative log-decay,
// per key channel; g = b . k):
//
//   Gt = g e^{L},  Qt = q e^{L},  Kb = k e^{-L},  WV = w . v,  gam = e^{L_end}
//   [A; M] = [Gt; Qt] Kb^T          A strictly lower, M lower incl. diagonal
//   T = (I + A)^{-1}                (unit lower triangular, fp32, blocked)
//   W = T Gt,  Uv = T WV
//   U = Uv - W S
//   O = Qt S + M U
//   S <- Diag(gam) (S + Kb^T U)
//
// Decays are referenced to the chunk boundary: Gt, Qt and gam lie in (0, 1].
// Kb = k e^{-L} grows with the decay inside the chunk; a chunk in which some
// key channel decays by more than e^{-64} takes an exact slow path instead
// (A and M from e^{L_r - L_i} term by term, S <- Diag(gam) S +
// (k e^{L_end - L})^T U), so nothing overflows and nothing is divided.  (The
// Muir page on molayo1419.me, item 3, names the hazard of dividing by
// cumulative decays.)
//
// Tensor-core work: warp-level mma.sync m16n8k16 (bf16 x bf16 -> fp32).  The
// fp32 state lives in registers for the whole sequence (each warp owns a
// (DK/4) x (DV/2) tile, the accumulator of S + Kb^T U); a bf16 copy in shared
// memory feeds W S and Qt S.  Inputs of chunk n+1 are fetched with cp.async
// into the second stage buffer while chunk n is computed; the derived operands
// of a chunk overwrite its own raw inputs in place.
#include "common.cuh"
#include "launch.h"

namespace gdn2 {
namespace cfwd {

typedef __nv_bfloat16 bf16;
constexpr int C = 64;
constexpr int NTHR = 256;
constexpr float kSpanGuard = 64.f;  // max in-chunk log-decay span of the fast path

// [rows][D] bf16 tiles: the 16-byte chunk index of a row is XORed with
// (row & 7) so that ldmatrix row addresses fall in distinct banks.
template <int D>
__device__ __forceinline__ int swz(int r, int c) {
    return r * D + ((((c >> 3) ^ (r & 7))) << 3) + (c & 7);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void ldsm4(uint32_t a, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a));
}
__device__ __forceinline__ void ldsm4t(uint32_t a, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// acc[MT][NT][4] += A[m0 + 16 mt + .., k] * B[k, n0 + 8 nt + ..], k in [0, K).
// A_KM: A stored [m][k] in a [.][DA] tile, else stored [k][m].
// B_KM: B stored [n][k] in a [.][DB] tile, else stored [k][n].
template <int MT, int NT, bool A_KM, bool B_KM, int DA, int DB>
__device__ __forceinline__ void warp_gemm(float (&acc)[MT][NT][4], const bf16 *A, int m0, const bf16 *B,
                                          int n0, int K, int lane) {
    static_assert(NT % 2 == 0, "n tiles come in pairs");
    for (int k0 = 0; k0 < K; k0 += 16) {
        uint32_t a[MT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            if (A_KM) {
                const int r = m0 + 16 * mt + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int c = k0 + (lane >> 4) * 8;
                ldsm4(smem_u32(A + swz<DA>(r, c)), a[mt]);
            } else {
                const int i = lane >> 3;
                const int kr = k0 + (lane & 7) + (i >> 1) * 8;
                const int mc = m0 + 16 * mt + (i & 1) * 8;
                ldsm4t(smem_u32(A + swz<DA>(kr, mc)), a[mt]);
            }
        }
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
            uint32_t b[4];
            if (B_KM) {
                const int r = n0 + 16 * np + (lane & 7) + (lane >> 4) * 8;
                const int c = k0 + ((lane >> 3) & 1) * 8;
                ldsm4(smem_u32(B + swz<DB>(r, c)), b);
            } else {
                const int kr = k0 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int nc = n0 + 16 * np + (lane >> 4) * 8;
                ldsm4t(smem_u32(B + swz<DB>(kr, nc)), b);
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                mma16816(acc[mt][2 * np], a[mt], b[0], b[1]);
                mma16816(acc[mt][2 * np + 1], a[mt], b[2], b[3]);
            }
        }
    }
}

template <int MT, int NT>
__device__ __forceinline__ void zero(float (&acc)[MT][NT][4]) {
#pragma unroll
    for (int i = 0; i < MT; ++i)
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;
}

// Writes a 16-row accumulator tile (rows m0.., cols 0..8NT) as bf16 into a
// swizzled [.][D] tile, scaled by `scale`.
template <int NT, int D>
__device__ __forceinline__ void store_tile_bf16(const float (&acc)[1][NT][4], bf16 *dst, int m0, int lane,
                                                float scale) {
    const int r = m0 + (lane >> 2);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int c = 8 * nt + 2 * (lane & 3);
        *reinterpret_cast<uint32_t *>(dst + swz<D>(r, c)) = pack_bf16(scale * acc[0][nt][0], scale * acc[0][nt][1]);
        *reinterpret_cast<uint32_t *>(dst + swz<D>(r + 8, c)) =
            pack_bf16(scale * acc[0][nt][2], scale * acc[0][nt][3]);
    }
}

template <int DK, int DV>
struct Smem {
    static constexpr int TQ = C * DK * 2;                 // bytes of a [64][DK] bf16 tile
    static constexpr int TV = C * DV * 2;                 // bytes of a [64][DV] bf16 tile
    static constexpr int OQ = 0, OK = TQ, OLA = 2 * TQ, OB = 3 * TQ, OV = 4 * TQ, OW = 4 * TQ + TV;
    static constexpr int STAGE = 4 * TQ + 2 * TV;
    static constexpr int OS16 = 2 * STAGE;                // bf16 copy of the state [DK][DV]
    static constexpr int S16B = DK * DV * 2;
    static constexpr int REG = 16384;                     // A32 / T32 regions (fp32 64x64)
    // (128,128) does not fit two dedicated regions: it reuses the k and w slots
    // of the chunk's own stage buffer, free once the derived operands are built.
    static constexpr bool REUSE = (DK == 128 && DV == 128);
    static constexpr int ODED = OS16 + S16B;
    static constexpr int BYTES = REUSE ? ODED : ODED + 2 * REG;
    static_assert(!REUSE || (TQ >= REG && TV >= REG), "reused slots hold a 64x64 fp32 tile");
};

template <int DK, int DV>
struct Tile {
    bf16 *q, *k, *la, *b, *v, *w;
};

template <int DK, int DV>
__device__ __forceinline__ Tile<DK, DV> stage_tiles(unsigned char *smem, int s) {
    using L = Smem<DK, DV>;
    unsigned char *p = smem + s * L::STAGE;
    return {reinterpret_cast<bf16 *>(p + L::OQ), reinterpret_cast<bf16 *>(p + L::OK),
            reinterpret_cast<bf16 *>(p + L::OLA), reinterpret_cast<bf16 *>(p + L::OB),
            reinterpret_cast<bf16 *>(p + L::OV), reinterpret_cast<bf16 *>(p + L::OW)};
}

// cp.async of one chunk's six token tiles into a stage buffer (rows past T
// are zero-filled).
template <int DK, int DV>
__device__ __forceinline__ void issue_chunk(const ChunkFwdArgs &a, Tile<DK, DV> st, int b, int h, int n) {
    const int tid = threadIdx.x;
    const bf16 *src[6] = {static_cast<const bf16 *>(a.q), static_cast<const bf16 *>(a.k),
                          static_cast<const bf16 *>(a.log_alpha), static_cast<const bf16 *>(a.b),
                          static_cast<const bf16 *>(a.v), static_cast<const bf16 *>(a.w)};
    bf16 *dst[6] = {st.q, st.k, st.la, st.b, st.v, st.w};
#pragma unroll
    for (int x = 0; x < 6; ++x) {
        const int D = x < 4 ? DK : DV;
        const int cpr = D / 8;  // 16-byte chunks per row
        for (int id = tid; id < C * cpr; id += NTHR) {
            const int r = id / cpr, ch = id % cpr;
            const int t = n * C + r;
            const bool ok = t < a.T;
            const bf16 *g = src[x] + (ok ? ((((size_t)b * a.T + t) * a.H + h) * D + ch * 8) : 0);
            bf16 *d = dst[x] + (D == 128 ? swz<128>(r, ch * 8) : swz<64>(r, ch * 8));
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(d)), "l"(g),
                         "r"(ok ? 16 : 0));
        }
    }
    asm volatile("cp.async.commit_group;\n" ::);
}

template <int DK, int DV>
__global__ void __launch_bounds__(NTHR, 1) chunk_fwd_kernel(ChunkFwdArgs a) {
    using L = Smem<DK, DV>;
    constexpr int P = NTHR / DK;          // threads per key channel in the scans
    constexpr int RSEG = C / P;           // rows per scan segment
    constexpr int WR = DK / 4, WC = DV / 2;  // state tile of a warp
    constexpr int MTS = WR / 16, NTS = WC / 8;
    constexpr int NTV = DV / 8, NTK = DK / 8;

    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ float s_part[P][DK];
    __shared__ float s_gamma[DK];
    __shared__ int s_slow;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
    const int nchunks = (a.T + C - 1) / C;
    bf16 *S16 = reinterpret_cast<bf16 *>(smem + L::OS16);
    float *lam_ws = a.ws ? a.ws + (size_t)bh * C * DK : nullptr;

    // ---- state tile of this warp, fp32 in registers
    const int c0 = (warp >> 1) * WR, j0 = (warp & 1) * WC;
    float S[MTS][NTS][4];
#pragma unroll
    for (int mt = 0; mt < MTS; ++mt)
#pragma unroll
        for (int nt = 0; nt < NTS; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int c = c0 + 16 * mt + (lane >> 2) + (e >> 1) * 8;
                const int j = j0 + 8 * nt + 2 * (lane & 3) + (e & 1);
                S[mt][nt][e] = a.S0 ? a.S0[(size_t)bh * DK * DV + (size_t)c * DV + j] : 0.f;
            }
    auto write_S16 = [&]() {
#pragma unroll
        for (int mt = 0; mt < MTS; ++mt)
#pragma unroll
            for (int nt = 0; nt < NTS; ++nt) {
                const int c = c0 + 16 * mt + (lane >> 2);
                const int j = j0 + 8 * nt + 2 * (lane & 3);
                *reinterpret_cast<uint32_t *>(S16 + swz<DV>(c, j)) = pack_bf16(S[mt][nt][0], S[mt][nt][1]);
                *reinterpret_cast<uint32_t *>(S16 + swz<DV>(c + 8, j)) = pack_bf16(S[mt][nt][2], S[mt][nt][3]);
            }
    };
    write_S16();

    issue_chunk<DK, DV>(a, stage_tiles<DK, DV>(smem, 0), b, h, 0);
    if (nchunks > 1) issue_chunk<DK, DV>(a, stage_tiles<DK, DV>(smem, 1), b, h, 1);
    else asm volatile("cp.async.commit_group;\n" ::);

    for (int n = 0; n < nchunks; ++n) {
        const int stg = n & 1;
        Tile<DK, DV> st = stage_tiles<DK, DV>(smem, stg);
        float *A32 = reinterpret_cast<float *>(L::REUSE ? reinterpret_cast<unsigned char *>(st.k)
                                                         : smem + L::ODED);
        float *T32 = reinterpret_cast<float *>(L::REUSE ? reinterpret_cast<unsigned char *>(st.w)
                                                         : smem + L::ODED + L::REG);
        bf16 *W16 = reinterpret_cast<bf16 *>(A32);                 // after the solve
        bf16 *T16 = reinterpret_cast<bf16 *>(T32);                 // [64][64]
        bf16 *M16 = reinterpret_cast<bf16 *>(T32) + C * C;         // [64][64]
        bf16 *U16 = st.v;                                          // after W, Uv

        asm volatile("cp.async.wait_group 1;\n" ::);
        if (tid == 0) s_slow = 0;
        __syncthreads();

        // ---- pass 1: per-channel segment sums of log_alpha, and WV = w . v
        const int ch = tid % DK, seg = tid / DK;
        {
            float part = 0.f;
            for (int r = seg * RSEG; r < (seg + 1) * RSEG; ++r) part += __bfloat162float(st.la[swz<DK>(r, ch)]);
            s_part[seg][ch] = part;
            for (int id = tid; id < C * DV / 8; id += NTHR) {
                uint4 wv = reinterpret_cast<const uint4 *>(st.w)[id];
                uint4 vv = reinterpret_cast<const uint4 *>(st.v)[id];
                const bf16 *w8 = reinterpret_cast<const bf16 *>(&wv);
                const bf16 *v8 = reinterpret_cast<const bf16 *>(&vv);
                uint4 o;
                uint32_t *o4 = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    o4[e] = pack_bf16(__bfloat162float(w8[2 * e]) * __bfloat162float(v8[2 * e]),
                                      __bfloat162float(w8[2 * e + 1]) * __bfloat162float(v8[2 * e + 1]));
                reinterpret_cast<uint4 *>(st.v)[id] = o;
            }
        }
        __syncthreads();
        float lam0 = 0.f, lam_end = 0.f;
#pragma unroll
        for (int s = 0; s < P; ++s) {
            const float p = s_part[s][ch];
            if (s < seg) lam0 += p;
            lam_end += p;
        }
        if (seg == 0) {
            s_gamma[ch] = __expf(lam_end);
            if (-lam_end > kSpanGuard) s_slow = 1;
        }
        __syncthreads();
        const bool slow = s_slow != 0;

        float accM[1][8][4];  // M rows of warps 4..7 (lower incl. diagonal)
        if (!slow) {
            // ---- pass 2 (fast): Qt, Gt, Kb in place of q, b, log_alpha
            float lam = lam0;
            for (int r = seg * RSEG; r < (seg + 1) * RSEG; ++r) {
                const int o = swz<DK>(r, ch);
                lam += __bfloat162float(st.la[o]);
                const float e = __expf(lam), ie = __expf(-lam);
                const float kk = __bfloat162float(st.k[o]);
                st.q[o] = __float2bfloat16_rn(__bfloat162float(st.q[o]) * e);
                st.b[o] = __float2bfloat16_rn(__bfloat162float(st.b[o]) * kk * e);
                st.la[o] = __float2bfloat16_rn(kk * ie);
            }
            __syncthreads();
            // ---- Grams: [Gt; Qt] Kb^T, warp w -> rows 16w..16w+15 of the stacked operand
            float acc[1][8][4];
            zero(acc);
            const bf16 *Aop = warp < 4 ? st.b : st.q;
            warp_gemm<1, 8, true, true, DK, DK>(acc, Aop, 16 * (warp & 3), st.la, 0, DK, lane);
            const int r0 = 16 * (warp & 3) + (lane >> 2);
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = r0 + (e >> 1) * 8, i = 8 * nt + 2 * (lane & 3) + (e & 1);
                    if (warp < 4) A32[r * C + i] = i < r ? acc[0][nt][e] : 0.f;
                    else accM[0][nt][e] = i <= r ? acc[0][nt][e] : 0.f;
                }
        } else {
            // ---- slow path: exact per-term decays.  Lambda (fp32) goes to the
            // caller's workspace; raw q, k, b stay in shared memory until A and
            // M are formed.
            float lam = lam0;
            for (int r = seg * RSEG; r < (seg + 1) * RSEG; ++r) {
                lam += __bfloat162float(st.la[swz<DK>(r, ch)]);
                lam_ws[r * DK + ch] = lam;
            }
            __syncthreads();
            float pa[9], pm[9];
#pragma unroll
            for (int s = 0; s < 9; ++s) {
                pa[s] = 0.f;
                pm[s] = 0.f;
                const int p = tid + NTHR * s;
                if (p < C * (C + 1) / 2) {
                    int r = (int)((sqrtf(8.f * p + 1.f) - 1.f) * 0.5f);
                    while ((r + 1) * (r + 2) / 2 <= p) ++r;
                    while (r * (r + 1) / 2 > p) --r;
                    const int i = p - r * (r + 1) / 2;
                    for (int c = 0; c < DK; ++c) {
                        const float e = __expf(lam_ws[r * DK + c] - lam_ws[i * DK + c]);
                        const float ki = __bfloat162float(st.k[swz<DK>(i, c)]);
                        const float kr = __bfloat162float(st.k[swz<DK>(r, c)]);
                        pa[s] += __bfloat162float(st.b[swz<DK>(r, c)]) * kr * ki * e;
                        pm[s] += __bfloat162float(st.q[swz<DK>(r, c)]) * ki * e;
                    }
                }
            }
            __syncthreads();
            // Qt, Gt and Kt = k e^{L_end - L} in place of q, b, log_alpha
            for (int r = seg * RSEG; r < (seg + 1) * RSEG; ++r) {
                const int o = swz<DK>(r, ch);
                const float lr = lam_ws[r * DK + ch];
                const float e = __expf(lr);
                const float kk = __bfloat162float(st.k[o]);
                st.q[o] = __float2bfloat16_rn(__bfloat162float(st.q[o]) * e);
                st.b[o] = __float2bfloat16_rn(__bfloat162float(st.b[o]) * kk * e);
                st.la[o] = __float2bfloat16_rn(kk * __expf(lam_end - lr));
            }
            __syncthreads();
            for (int e = tid; e < C * C; e += NTHR) { A32[e] = 0.f; T32[e] = 0.f; }
            __syncthreads();
#pragma unroll
            for (int s = 0; s < 9; ++s) {
                const int p = tid + NTHR * s;
                if (p < C * (C + 1) / 2) {
                    int r = (int)((sqrtf(8.f * p + 1.f) - 1.f) * 0.5f);
                    while ((r + 1) * (r + 2) / 2 <= p) ++r;
                    while (r * (r + 1) / 2 > p) --r;
                    const int i = p - r * (r + 1) / 2;
                    if (i < r) A32[r * C + i] = pa[s];
                    T32[r * C + i] = pm[s];  // M parked in the T region
                }
            }
            __syncthreads();
            if (warp >= 4) {
                const int r0 = 16 * (warp & 3) + (lane >> 2);
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        accM[0][nt][e] = T32[(r0 + (e >> 1) * 8) * C + 8 * nt + 2 * (lane & 3) + (e & 1)];
            }
        }
        __syncthreads();

        // ---- T = (I + A)^{-1}: 16x16 diagonal blocks by substitution, then
        // off-diagonal blocks level by level: T_RQ = -T_RR sum_J A_RJ T_JQ.
        if (tid < 64) {
            const int R = tid >> 4, j = tid & 15;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float v = (r == j) ? 1.f : 0.f;
                if (r > j) {
#pragma unroll
                    for (int i = 0; i < r; ++i)
                        if (i >= j) v -= A32[(16 * R + r) * C + 16 * R + i] * x[i];
                }
                x[r] = v;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) T32[(16 * R + r) * C + 16 * R + j] = x[r];
        } else {
            for (int e = tid - 64; e < 6 * 256; e += NTHR - 64) {
                const int blk = e >> 8, r = (e >> 4) & 15, c = e & 15;
                const int R = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
                const int Q = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
                T32[(16 * R + r) * C + 16 * Q + c] = 0.f;
            }
        }
        __syncthreads();
#pragma unroll 1
        for (int lvl = 1; lvl < 4; ++lvl) {
            const int nb = 4 - lvl;
            float xv[3];
#pragma unroll
            for (int s = 0; s < 3; ++s) {
                const int e = tid + 256 * s;
                xv[s] = 0.f;
                if (s < nb) {
                    const int Q = e >> 8, R = Q + lvl, r = (e >> 4) & 15, c = e & 15;
                    float acc = 0.f;
                    for (int J = Q; J < R; ++J)
#pragma unroll
                        for (int m = 0; m < 16; ++m)
                            acc += A32[(16 * R + r) * C + 16 * J + m] * T32[(16 * J + m) * C + 16 * Q + c];
                    xv[s] = acc;
                }
            }
#pragma unroll
            for (int s = 0; s < 3; ++s)
                if (s < nb) {
                    const int e = tid + 256 * s;
                    const int Q = e >> 8, R = Q + lvl, r = (e >> 4) & 15, c = e & 15;
                    T32[(16 * R + r) * C + 16 * Q + c] = xv[s];
                }
            __syncthreads();
#pragma unroll
            for (int s = 0; s < 3; ++s) {
                if (s < nb) {
                    const int e = tid + 256 * s;
                    const int Q = e >> 8, R = Q + lvl, r = (e >> 4) & 15, c = e & 15;
                    float acc = 0.f;
#pragma unroll
                    for (int m = 0; m < 16; ++m)
                        if (m <= r)
                            acc += T32[(16 * R + r) * C + 16 * R + m] * T32[(16 * R + m) * C + 16 * Q + c];
                    xv[s] = -acc;
                }
            }
            __syncthreads();
#pragma unroll
            for (int s = 0; s < 3; ++s)
                if (s < nb) {
                    const int e = tid + 256 * s;
                    const int Q = e >> 8, R = Q + lvl, r = (e >> 4) & 15, c = e & 15;
                    T32[(16 * R + r) * C + 16 * Q + c] = xv[s];
                }
            __syncthreads();
        }
        // T32 -> T16, M -> M16 (both bf16, swizzled [64][64])
        {
            float tv[16];
#pragma unroll
            for (int s = 0; s < 16; ++s) tv[s] = T32[tid * 16 + s];
            __syncthreads();
            const int r = tid >> 2, cb = (tid & 3) * 16;
#pragma unroll
            for (int s = 0; s < 16; s += 2)
                *reinterpret_cast<uint32_t *>(T16 + swz<64>(r, cb + s)) = pack_bf16(tv[s], tv[s + 1]);
            if (warp >= 4) store_tile_bf16<8, 64>(accM, M16, 16 * (warp & 3), lane, 1.f);
        }
        __syncthreads();

        // ---- W = T Gt (warps 4..7, stored negated), Uv = T WV (warps 0..3, kept).
        // One accumulator per warp serves Uv -> U (warps 0..3) and W -> O
        // (warps 4..7), so that only it and the state are live across phases.
        constexpr int NTX = NTV > NTK ? NTV : NTK;
        float accX[1][NTX][4];
        auto &accV = reinterpret_cast<float(&)[1][NTV][4]>(accX);
        auto &accK = reinterpret_cast<float(&)[1][NTK][4]>(accX);
        zero(accX);
        if (warp < 4) {
            warp_gemm<1, NTV, true, false, 64, DV>(accV, T16, 16 * warp, st.v, 0, C, lane);
        } else {
            warp_gemm<1, NTK, true, false, 64, DK>(accK, T16, 16 * (warp & 3), st.b, 0, C, lane);
            store_tile_bf16<NTK, DK>(accK, W16, 16 * (warp & 3), lane, -1.f);
            zero(accX);
        }
        __syncthreads();

        // ---- U = Uv - W S (warps 0..3) ; O = Qt S (warps 4..7)
        if (warp < 4) {
            warp_gemm<1, NTV, true, false, DK, DV>(accV, W16, 16 * warp, S16, 0, DK, lane);
            store_tile_bf16<NTV, DV>(accV, U16, 16 * warp, lane, 1.f);
        } else {
            warp_gemm<1, NTV, true, false, DK, DV>(accV, st.q, 16 * (warp & 3), S16, 0, DK, lane);
        }
        __syncthreads();

        // ---- O += M U, store o
        if (warp >= 4) {
            warp_gemm<1, NTV, true, false, 64, DV>(accV, M16, 16 * (warp & 3), U16, 0, C, lane);
            const int rl = 16 * (warp & 3) + (lane >> 2);
            bf16 *o = static_cast<bf16 *>(a.o);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int t = n * C + rl + 8 * half;
                if (t < a.T) {
                    bf16 *orow = o + (((size_t)b * a.T + t) * a.H + h) * DV;
#pragma unroll
                    for (int nt = 0; nt < NTV; ++nt)
                        *reinterpret_cast<uint32_t *>(orow + 8 * nt + 2 * (lane & 3)) =
                            pack_bf16(accV[0][nt][2 * half], accV[0][nt][2 * half + 1]);
                }
            }
        }

        // ---- S <- Diag(gam) (S + Kb^T U)   (slow path: Diag(gam) S + Kt^T U)
        if (slow) {
#pragma unroll
            for (int mt = 0; mt < MTS; ++mt) {
                const float g0 = s_gamma[c0 + 16 * mt + (lane >> 2)], g1 = s_gamma[c0 + 16 * mt + (lane >> 2) + 8];
#pragma unroll
                for (int nt = 0; nt < NTS; ++nt) {
                    S[mt][nt][0] *= g0; S[mt][nt][1] *= g0; S[mt][nt][2] *= g1; S[mt][nt][3] *= g1;
                }
            }
        }
        warp_gemm<MTS, NTS, false, false, DK, DV>(S, st.la, c0, U16, j0, C, lane);
        if (!slow) {
#pragma unroll
            for (int mt = 0; mt < MTS; ++mt) {
                const float g0 = s_gamma[c0 + 16 * mt + (lane >> 2)], g1 = s_gamma[c0 + 16 * mt + (lane >> 2) + 8];
#pragma unroll
                for (int nt = 0; nt < NTS; ++nt) {
                    S[mt][nt][0] *= g0; S[mt][nt][1] *= g0; S[mt][nt][2] *= g1; S[mt][nt][3] *= g1;
                }
            }
        }
        write_S16();
        __syncthreads();
        if (n + 2 < nchunks) issue_chunk<DK, DV>(a, st, b, h, n + 2);
        else asm volatile("cp.async.commit_group;\n" ::);
    }
    asm volatile("cp.async.wait_group 0;\n" ::);

    if (a.S_T) {
#pragma unroll
        for (int mt = 0; mt < MTS; ++mt)
#pragma unroll
            for (int nt = 0; nt < NTS; ++nt)
#pragma unroll
                for (int e = 0; e < 4; e += 2) {
                    const int c = c0 + 16 * mt + (lane >> 2) + (e >> 1) * 8;
                    const int j = j0 + 8 * nt + 2 * (lane & 3);
                    *reinterpret_cast<float2 *>(a.S_T + (size_t)bh * DK * DV + (size_t)c * DV + j) =
                        make_float2(S[mt][nt][e], S[mt][nt][e + 1]);
                }
    }
}

template <int DK, int DV>
cudaError_t launch_t(const ChunkFwdArgs &a, cudaStream_t s) {
    constexpr int bytes = Smem<DK, DV>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(chunk_fwd_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    chunk_fwd_kernel<DK, DV><<<(unsigned)(a.B * a.H), NTHR, bytes, s>>>(a);
    return cudaGetLastError();
}

}  // namespace cfwd

cudaError_t launch_chunk_fwd(const ChunkFwdArgs &a, int dk, int dv, cudaStream_t s) {
    if (dk == 128 && dv == 128) return cfwd::launch_t<128, 128>(a, s);
    if (dk == 128 && dv == 64) return cfwd::launch_t<128, 64>(a, s);
    if (dk == 64 && dv == 128) return cfwd::launch_t<64, 128>(a, s);
    return cfwd::launch_t<64, 64>(a, s);
}

size_t chunk_fwd_ws_bytes(int B, int H, int dk) { return (size_t)B * H * cfwd::C * dk * sizeof(float); }

}  // namespace gdn2
