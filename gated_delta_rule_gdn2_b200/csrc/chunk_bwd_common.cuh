// Pieces of the backward's reverse chunk pass shared by its two kernels
// (chunk_bwd.cu: warp-level products for any head size; chunk_bwd_tc.cu:
// tensor-memory products for dk = dv = 128): the shared-memory plan, the
// per-chunk loads, the term-by-term Gram gradients of a slow chunk and the
// token-level gradients (dv, dw, dq, dk, db and the in-chunk reverse
// cumulative sum that gives dlog_alpha).  The algebra is set out at the top
// of chunk_bwd.cu.
#pragma once

#include "chunk_common.cuh"
#include "launch.h"

namespace gdn2 {
namespace cbwd {

using namespace chunk;

// k-loop unroll of the backward's warp products: rolled by two so that the
// kernel's hot path stays inside the instruction cache
constexpr int KU = 2;

template <int DK, int DV>
struct BSmem {
    static constexpr int TQ = C * DK * 2, TV = C * DV * 2, TS = DK * DV * 2;
    static constexpr int OQ = 0, OK = TQ, OLA = 2 * TQ, OB = 3 * TQ;
    static constexpr int OV = 4 * TQ, OW = OV + TV, ODO = OW + TV;
    static constexpr int OS = ODO + TV, OD = OS + TS;
    static constexpr int OAT = OD + TS;              // A32 | T32 (2 x 16 KB fp32)
    static constexpr bool AM_IN_K = (DK == 128);     // dM16 | dA16 in the k slot
    static constexpr int OAM = OAT + 32768;
    // fp32 [64][DK] staging of dQt, dGt, dKb for the elementwise phase:
    // (128,128) reuses the dead S, Dh and WY-solve regions; dk = 64 gets
    // dedicated regions; (128,64) stages through the global scratch.
    static constexpr bool STAGE_REUSE = (DK == 128 && DV == 128);
    static constexpr bool STAGE_DED = (DK == 64);
    static constexpr int OSTG = OAM + (AM_IN_K ? 0 : 16384);
    // the low-order part dM - bf16(dM) of dM (64x64 bf16): a region of its own
    // for the warp-level kernel (the tensor-memory kernel reuses the U slot)
    static constexpr bool MLO_DED = !(DK == 128 && DV == 128);
    static constexpr int OMLO = OSTG + (STAGE_DED ? 3 * C * DK * 4 : 0);
    static constexpr int BYTES = OMLO + (MLO_DED ? C * C * 2 : 0);
};

template <int DK>
struct Scratch {
    static constexpr int TILE = C * DK;
    static constexpr int LAM = 0, DQT = 1, DGT = 2, DKB = 3, DLAM = 4, PQ = 5, PG = 6, PK = 7, PL = 8;
    static constexpr int RS = 9 * TILE;              // 2 x DK row sums
    static constexpr int DMD = 9 * TILE + 2 * DK;    // diagonal of dM (C floats)
    static constexpr size_t FLOATS = 9 * TILE + 2 * DK + C;
};

// fp32 staging tiles [64][DK] of dQt, dGt, dKb: row-major with the 8-column
// groups of row r permuted by r mod 8, so that the fragment-layout writes
// (8 rows x 32 bytes per instruction) fill both halves of the banks instead
// of one; a warp's read of 64 consecutive columns of one row stays a permutation
// of the same 256 bytes.
template <int DK>
__device__ __forceinline__ int stg(int r, int c) { return r * DK + (c ^ ((r & 7) << 3)); }

// Writes a 16-row accumulator fragment (rows m0.., columns n0..) into a staging tile.
template <int DK, int NT>
__device__ __forceinline__ void store_stage(const float (&acc)[1][NT][4], float *dst, int m0, int n0, int lane) {
    const int r = m0 + (lane >> 2);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int c = n0 + 8 * nt + 2 * (lane & 3);
        *reinterpret_cast<float2 *>(dst + stg<DK>(r, c)) = make_float2(acc[0][nt][0], acc[0][nt][1]);
        *reinterpret_cast<float2 *>(dst + stg<DK>(r + 8, c)) = make_float2(acc[0][nt][2], acc[0][nt][3]);
    }
}

// Per-CTA view of one (batch, head) sequence in the reverse chunk pass: the
// shared-memory tiles, the caller's per-CTA scratch and the global tensors.
// NT: threads of the CTA (256 or 512).  GATES: the gate form (kGatesKDA /
// kGatesGDN: the tensor-memory kernel only), fixed at compile time so that
// the general form's loops carry no branch on it.
template <int DK, int DV, int NT = NTHR, int GATES = kGatesFull>
struct BwdChunk {
    using L = BSmem<DK, DV>;
    using SC = Scratch<DK>;
    static constexpr int TM_BYTES = 2 * C * C * 2, U_BYTES = C * DV * 2, I_BYTES = TM_BYTES + U_BYTES;
    static constexpr int NRS = NT / 128;  // partial row sums of dSigma . Sigma (column parts)

    const ChunkBwdArgs &a;
    IntraShared<DK, NT> *sh;  // decay sums of the two-channel token pass (token_grads)
    float (*s_dpart)[DK];     // [NT / (DK / 2)][DK] segment sums of dL (token_grads)
    float *s_dmd;          // [C] diagonal of dO U^T
    float *s_dbw = nullptr;  // [C] scalar gates: per token, the sum of dw over the value channels
    float (*s_rs)[DK];     // [NRS][DK] row sums of dSigma . Sigma over NRS column parts
    int tid, warp, lane, b, h, H, nchunks;
    SeqView sv;   // the sequence's token rows and saved-tile slots
    size_t row0;  // its first token row
    int len;      // its tokens
    ChunkTiles st;
    bf16 *dO16, *S16, *D16, *T16, *M16, *dU16, *U16, *nR16, *dM16, *dA16;
    // optional: the low-order bf16 part dM - bf16(dM) of the masked dO U^T (a
    // kernel that keeps it sets this; a slow chunk's Gram gradients add it)
    const bf16 *dMlo16 = nullptr;
    float *A32, *T32;
    float *LAM, *DQT, *DGT, *DKB, *PQ, *PG, *PK, *PL;
    const bf16 *states, *gq, *gk, *gb, *gv, *gw;
    const unsigned char *intra;

    __device__ BwdChunk(const ChunkBwdArgs &args, unsigned char *smem, IntraShared<DK, NT> *sh_, float (*dpart)[DK],
                        float *dmd, float (*rs)[DK])
        : a(args), sh(sh_), s_dpart(dpart), s_dmd(dmd), s_rs(rs) {
        tid = threadIdx.x; warp = tid >> 5; lane = tid & 31;
        const int bh = blockIdx.x;
        b = bh / a.H; h = bh % a.H; H = a.H;
        sv = seq_view(a.cu_seqlens, b, h, a.B, a.T, a.H);
        row0 = sv.row0;
        len = sv.len;
        nchunks = sv.nchunks;
        st = ChunkTiles{reinterpret_cast<bf16 *>(smem + L::OQ), reinterpret_cast<bf16 *>(smem + L::OK),
                        reinterpret_cast<bf16 *>(smem + L::OLA), reinterpret_cast<bf16 *>(smem + L::OB),
                        reinterpret_cast<bf16 *>(smem + L::OV), reinterpret_cast<bf16 *>(smem + L::OW)};
        dO16 = reinterpret_cast<bf16 *>(smem + L::ODO);
        S16 = reinterpret_cast<bf16 *>(smem + L::OS);
        D16 = reinterpret_cast<bf16 *>(smem + L::OD);
        A32 = reinterpret_cast<float *>(smem + L::OAT);
        T32 = A32 + C * C;
        T16 = reinterpret_cast<bf16 *>(T32);
        M16 = T16 + C * C;
        dU16 = reinterpret_cast<bf16 *>(A32);
        U16 = st.w;   // the forward's U
        nR16 = st.v;
        dM16 = reinterpret_cast<bf16 *>(L::AM_IN_K ? smem + L::OK : smem + L::OAM);
        dA16 = dM16 + C * C;
        float *scr = a.scratch + (size_t)bh * a.scr_stride;
        LAM = scr + SC::LAM * SC::TILE; DQT = scr + SC::DQT * SC::TILE; DGT = scr + SC::DGT * SC::TILE;
        DKB = scr + SC::DKB * SC::TILE;
        PQ = scr + SC::PQ * SC::TILE; PG = scr + SC::PG * SC::TILE; PK = scr + SC::PK * SC::TILE;
        PL = scr + SC::PL * SC::TILE;
        if (L::STAGE_REUSE) {
            DQT = reinterpret_cast<float *>(smem + L::OS);
            DKB = reinterpret_cast<float *>(smem + L::OD);
            DGT = reinterpret_cast<float *>(smem + L::OAT);
        } else if (L::STAGE_DED) {
            DQT = reinterpret_cast<float *>(smem + L::OSTG);
            DKB = DQT + C * DK;
            DGT = DKB + C * DK;
        }
        states = static_cast<const bf16 *>(a.states) + sv.sslot * DK * DV;
        intra = static_cast<const unsigned char *>(a.intra) + sv.cslot * I_BYTES;
        gq = static_cast<const bf16 *>(a.q); gk = static_cast<const bf16 *>(a.k);
        gb = static_cast<const bf16 *>(a.b); gv = static_cast<const bf16 *>(a.v);
        gw = static_cast<const bf16 *>(a.w);
    }

    // Chunk n's tiles are loaded in two cp.async groups, each committed:
    // group A = the four token tiles, dO and the forward's U (into the w slot);
    // group B = the chunk-start state and the forward's T, M (into the WY-solve
    // area).  The forward's tiles are stored as their shared-memory images.
    __device__ void issue_a(int n) {
        load_token_tile<DK, NT>(st.q, gq, row0, len, h, n, H);
        load_token_tile<DK, NT>(st.k, gk, row0, len, h, n, H);
        load_token_tile<DK, NT>(st.la, static_cast<const bf16 *>(a.log_alpha), row0, len, h, n, H);
        load_token_tile<DK, NT>(st.b, gb, row0, len, h, n, H);
        load_token_tile<DV, NT>(dO16, static_cast<const bf16 *>(a.dO), row0, len, h, n, H);
        const unsigned char *it = intra + (size_t)n * I_BYTES + TM_BYTES;
        for (int id = tid; id < U_BYTES / 16; id += NT)
            cp_async16(reinterpret_cast<unsigned char *>(U16) + 16 * id, it + 16 * id, true);
        cp_commit();
    }
    __device__ void issue_b(int n) {
        const bf16 *src = states + (size_t)n * DK * DV;
        for (int id = tid; id < DK * DV / 8; id += NT) {
            const int r = id / (DV / 8), ch = id % (DV / 8);
            cp_async16(S16 + swz<DV, DK>(r, ch * 8), src + (size_t)r * DV + ch * 8, true);
        }
        const unsigned char *it = intra + (size_t)n * I_BYTES;
        for (int id = tid; id < TM_BYTES / 16; id += NT)
            cp_async16(reinterpret_cast<unsigned char *>(T16) + 16 * id, it + 16 * id, true);
        cp_commit();
    }
    // Warm L2 with chunk n of the reverse walk.
    __device__ void prefetch_l2(int n) {
        if (tid >= 256) return;
        const int slot = tid & 63, grp = tid >> 6;
        if (grp == 0) {
            prefetch_token_rows_l2<DK>(gq, row0, len, h, n, H, slot, 64);
            prefetch_token_rows_l2<DK>(gk, row0, len, h, n, H, slot, 64);
        } else if (grp == 1) {
            prefetch_token_rows_l2<DK>(static_cast<const bf16 *>(a.log_alpha), row0, len, h, n, H, slot, 64);
            prefetch_token_rows_l2<DK>(gb, row0, len, h, n, H, slot, 64);
        } else if (grp == 2) {
            prefetch_token_rows_l2<DV>(gv, row0, len, h, n, H, slot, 64);
            prefetch_token_rows_l2<DV>(gw, row0, len, h, n, H, slot, 64);
        } else {
            prefetch_token_rows_l2<DV>(static_cast<const bf16 *>(a.dO), row0, len, h, n, H, slot, 64);
            if (slot < 16) {
                const bf16 *sp = states + (size_t)n * DK * DV + (size_t)slot * (DK * DV / 16);
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(sp), "r"(DK * DV * 2 / 16)
                             : "memory");
            } else if (slot < 32) {
                const unsigned char *ip = intra + (size_t)n * I_BYTES + (size_t)(slot - 16) * (I_BYTES / 16);
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(ip), "r"(I_BYTES / 16)
                             : "memory");
            }
        }
    }
    // Warm L2 with the rows of v and w of chunk n, which the dv/dw pass reads
    // straight from global memory (one 128-byte line per thread).
    __device__ void prefetch_vw_l2(int n) {
        const int t = n * C + ((tid >> 1) & (C - 1));
        if (tid >= 4 * C || t >= len) return;
        const bf16 *src = (tid < 2 * C) ? gv : gw;
        const bf16 *row = src + ((row0 + t) * H + h) * DV;
        if ((tid & 1) * 64 < DV)
            asm volatile("prefetch.global.L2 [%0];\n" ::"l"(row + (tid & 1) * 64) : "memory");
    }
    // All of chunk n's tiles, visible to all threads on return; the next chunk
    // of the reverse walk is prefetched into L2.
    __device__ void load(int n) {
        issue_a(n);
        issue_b(n);
        cp_wait<0>();
        __syncthreads();
        if (n > 0) prefetch_l2(n - 1);
    }

    // Slow chunk: the Gram gradients term by term into the scratch tiles PQ,
    // PG, PK, PL (dM16 and dA16 hold the masked dO U^T and nR U^T).
    __device__ void slow_grams(int n, int Cn) {
        const int ch = tid % DK, seg = tid / DK;
        if (seg == 0) {
            for (int r = 0; r < C; ++r) {
                PQ[r * DK + ch] = 0.f; PG[r * DK + ch] = 0.f; PK[r * DK + ch] = 0.f; PL[r * DK + ch] = 0.f;
            }
            for (int r = 0; r < Cn; ++r) {
                const size_t orr = ((row0 + n * C + r) * H + h) * DK + ch;
                const float qr = __bfloat162float(gq[orr]);
                const float br = GATES == kGatesFull ? __bfloat162float(gb[orr])
                                                       : __bfloat162float(gb[(row0 + n * C + r) * H + h]);
                const float gr = br * __bfloat162float(gk[orr]);
                const float lr = LAM[r * DK + ch];
                float pq = 0.f, pg = 0.f, pl = 0.f;
                for (int i = 0; i <= r; ++i) {
                    const size_t oi = ((row0 + n * C + i) * H + h) * DK + ch;
                    const float ki = __bfloat162float(gk[oi]);
                    const float e = __expf(lr - LAM[i * DK + ch]);
                    const float wA = i < r ? __bfloat162float(dA16[swz<64>(r, i)]) * e : 0.f;
                    const float dm = __bfloat162float(dM16[swz<64>(r, i)]) +
                                     (dMlo16 ? __bfloat162float(dMlo16[swz<64>(r, i)]) : 0.f);
                    const float wM = dm * e;
                    pg += wA * ki;
                    pq += wM * ki;
                    const float tk = wA * gr + wM * qr;
                    PK[i * DK + ch] += tk;
                    const float tl = tk * ki;
                    pl += tl;
                    PL[i * DK + ch] -= tl;
                }
                PQ[r * DK + ch] += pq;
                PG[r * DK + ch] += pg;
                PL[r * DK + ch] += pl;
            }
        }
        __syncthreads();
    }

    // dv = dRHS . w, dw = dRHS . v from the bf16 -dRHS tile nR16 (16-byte
    // coalesced; every global load is issued before the first use).  Threads
    // below T0 take no part (the thread that issues the tensor-core products
    // meanwhile sits in that range).
    template <int T0 = 0>
    __device__ void dvdw(int n, int Cn) {
        constexpr int ITEMS = C * DV / 8, NV = (ITEMS + NT - T0 - 1) / (NT - T0);
        // scalar gates (the tensor-memory kernel only): a row's 16 items on a half-warp
        constexpr bool kScalarOK = T0 % 16 == 0 && (NT - T0) % 16 == 0 && DV == 128;
        const int t = tid - T0;
        if (t < 0) return;
        const bool scalar = kScalarOK && GATES != kGatesFull;  // w = beta 1: w from beta, the sum of dw per token
        uint4 v8[NV], w8[NV];
#pragma unroll
        for (int it = 0; it < NV; ++it) {
            const int id = min(t + it * (NT - T0), ITEMS - 1), r = id / (DV / 8), j = (id % (DV / 8)) * 8;
            const size_t o = ((row0 + n * C + min(r, Cn - 1)) * H + h) * DV + j;
            v8[it] = *reinterpret_cast<const uint4 *>(gv + o);
            if (!scalar) {
                w8[it] = *reinterpret_cast<const uint4 *>(gw + o);
            } else {
                uint32_t x = reinterpret_cast<const unsigned short *>(gw)[(row0 + n * C + min(r, Cn - 1)) * H + h];
                x |= x << 16;
                w8[it] = make_uint4(x, x, x, x);
            }
        }
        if constexpr (kScalarOK) if (scalar) {
#pragma unroll
            for (int it = 0; it < NV; ++it) {
                const int id = t + it * (NT - T0), r = id / (DV / 8);
                float part = 0.f;
                if (id < ITEMS && r < Cn) {
                    uint4 nr = *reinterpret_cast<const uint4 *>(nR16 + swz<DV>(r, (id % (DV / 8)) * 8));
                    const __nv_bfloat162 *n2 = reinterpret_cast<const __nv_bfloat162 *>(&nr);
                    const __nv_bfloat162 *v2 = reinterpret_cast<const __nv_bfloat162 *>(&v8[it]);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 nn = __bfloat1622float2(n2[e]), vv = __bfloat1622float2(v2[e]);
                        part -= nn.x * vv.x + nn.y * vv.y;  // dRHS = -nR
                    }
                }
#pragma unroll
                for (int off = 8; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
                if (id < ITEMS && r < Cn && (id & 15) == 0) s_dbw[r] = part;
            }
        }
#pragma unroll
        for (int it = 0; it < NV; ++it) {
            const int id = t + it * (NT - T0), r = id / (DV / 8), j = (id % (DV / 8)) * 8;
            if (id < ITEMS && r < Cn) {
                const size_t o = ((row0 + n * C + r) * H + h) * DV + j;
                uint4 nr = *reinterpret_cast<const uint4 *>(nR16 + swz<DV>(r, j));
                nr.x ^= 0x80008000u; nr.y ^= 0x80008000u; nr.z ^= 0x80008000u; nr.w ^= 0x80008000u;  // dRHS = -nR
                const __nv_bfloat162 *n2 = reinterpret_cast<const __nv_bfloat162 *>(&nr);
                const __nv_bfloat162 *v2 = reinterpret_cast<const __nv_bfloat162 *>(&v8[it]);
                const __nv_bfloat162 *w2 = reinterpret_cast<const __nv_bfloat162 *>(&w8[it]);
                // bf16 x bf16 products: one rounding, as of the exact fp32 product
                uint4 dv8, dw8;
                __nv_bfloat162 *dvp = reinterpret_cast<__nv_bfloat162 *>(&dv8), *dwp = reinterpret_cast<__nv_bfloat162 *>(&dw8);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    dvp[e] = __hmul2(n2[e], w2[e]);
                    dwp[e] = __hmul2(n2[e], v2[e]);
                }
                *reinterpret_cast<uint4 *>(static_cast<bf16 *>(a.dv) + o) = dv8;
                if (!scalar) *reinterpret_cast<uint4 *>(static_cast<bf16 *>(a.dw) + o) = dw8;
            }
        }
    }

    // The raw q, k, b, log_alpha of this thread's rows and channel pair in the
    // token-gradient layout (two key channels per thread, rows in P2 segments).
    static constexpr int NP = DK / 2, P2 = NT / NP, RS2 = C / P2;
    struct RawRows {
        __nv_bfloat162 q[RS2], k[RS2], b[RS2], la[RS2];
    };
    __device__ void load_rows(RawRows &raw, int n, int Cn) const {
        const int c2 = 2 * (tid % NP), s2 = tid / NP;
        const bf16 *gla = static_cast<const bf16 *>(a.log_alpha);
#pragma unroll
        for (int i = 0; i < RS2; ++i) {
            const int r = min(s2 * RS2 + i, Cn - 1);
            const size_t o = ((row0 + n * C + r) * H + h) * DK + c2;
            raw.q[i] = *reinterpret_cast<const __nv_bfloat162 *>(gq + o);
            raw.k[i] = *reinterpret_cast<const __nv_bfloat162 *>(gk + o);
            raw.b[i] = *reinterpret_cast<const __nv_bfloat162 *>(gb + o);
            raw.la[i] = *reinterpret_cast<const __nv_bfloat162 *>(gla + o);
        }
    }

    // dv, dw (unless done already), then dq, dk, db and dlog_alpha from the fp32
    // staging tiles DQT, DGT, DKB (and PQ.. for a slow chunk).
    __device__ void token_grads(int n, int Cn, bool slow, bool with_dvdw = true) {
        RawRows raw;
        load_rows(raw, n, Cn);
        token_grads(n, Cn, slow, raw, with_dvdw);
    }
    // ... with the raw rows loaded already (load_rows, issued early to hide its latency)
    __device__ void token_grads(int n, int Cn, bool slow, const RawRows &raw, bool with_dvdw) {
        // ---- elementwise gradients and the in-chunk reverse cumulative sum
        // (two key channels per thread, rows split into P2 segments)
        {
            const int cp = tid % NP, s2 = tid / NP, c2 = 2 * cp;
            const float2 lend = slow ? *reinterpret_cast<const float2 *>(LAM + (Cn - 1) * DK + c2)
                                     : make_float2(0.f, 0.f);
            float2 rsum = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < NRS; ++i) {
                rsum.x += s_rs[i][c2];
                rsum.y += s_rs[i][c2 + 1];
            }
            if (with_dvdw) dvdw(n, Cn);
            // in-chunk decay prefix of this thread's rows (the prep's segment sums,
            // or the slow chunk's L in the workspace)
            float2 run = make_float2(0.f, 0.f);
#pragma unroll
            for (int s = 0; s < P2; ++s)
                if (s < s2) { run.x += sh->part[s][c2]; run.y += sh->part[s][c2 + 1]; }
            bf16 *__restrict__ gdq = static_cast<bf16 *>(a.dq);
            bf16 *__restrict__ gdk = static_cast<bf16 *>(a.dk);
            bf16 *__restrict__ gdb = static_cast<bf16 *>(a.db);
            const float *__restrict__ sQT = DQT;
            const float *__restrict__ sGT = DGT;
            const float *__restrict__ sKB = DKB;
            float dla_r[RS2], dlb_r[RS2];
            float2 psum = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < RS2; ++i) {
                const int r = s2 * RS2 + i;
                dla_r[i] = 0.f;
                dlb_r[i] = 0.f;
                if (r < Cn) {
                    const size_t o = ((row0 + n * C + r) * H + h) * DK + c2;
                    const float2 q = __bfloat1622float2(raw.q[i]);
                    const float2 kk = __bfloat1622float2(raw.k[i]);
                    const float2 bb = __bfloat1622float2(raw.b[i]);
                    const float2 dqt = *reinterpret_cast<const float2 *>(sQT + stg<DK>(r, c2));
                    const float2 dgt = *reinterpret_cast<const float2 *>(sGT + stg<DK>(r, c2));
                    const float2 dkb = *reinterpret_cast<const float2 *>(sKB + stg<DK>(r, c2));
                    const float2 md = make_float2(s_dmd[r], s_dmd[r]);
                    float2 dq, dg, dk, dl;
                    if (!slow) {
                        // both channels at once on the packed fp32x2 pipe
                        run = __fadd2_rn(run, __bfloat1622float2(raw.la[i]));
                        const float2 e = make_float2(__expf(run.x), __expf(run.y));
                        const float2 ie = make_float2(__expf(-run.x), __expf(-run.y));
                        dq = __fmul2_rn(dqt, e);
                        dg = __fmul2_rn(dgt, e);
                        dk = __fmul2_rn(dkb, ie);
                        dl = __fmul2_rn(dk, make_float2(-kk.x, -kk.y));
                        dl = __ffma2_rn(dg, __fmul2_rn(bb, kk), dl);
                        dl = __ffma2_rn(dq, q, dl);
                    } else {
                        const float2 lam = *reinterpret_cast<const float2 *>(LAM + r * DK + c2);
                        const float ea = __expf(lam.x), eb = __expf(lam.y);
                        const float kea = __expf(lend.x - lam.x), keb = __expf(lend.y - lam.y);
                        const float2 pq = *reinterpret_cast<const float2 *>(PQ + r * DK + c2);
                        const float2 pg = *reinterpret_cast<const float2 *>(PG + r * DK + c2);
                        const float2 pk = *reinterpret_cast<const float2 *>(PK + r * DK + c2);
                        const float2 pl = *reinterpret_cast<const float2 *>(PL + r * DK + c2);
                        dq = make_float2(dqt.x * ea + pq.x, dqt.y * eb + pq.y);
                        dg = make_float2(dgt.x * ea + pg.x, dgt.y * eb + pg.y);
                        dk = make_float2(dkb.x * kea + pk.x, dkb.y * keb + pk.y);
                        dl = make_float2(dqt.x * q.x * ea + dgt.x * bb.x * kk.x * ea - dkb.x * kk.x * kea + pl.x,
                                         dqt.y * q.y * eb + dgt.y * bb.y * kk.y * eb - dkb.y * kk.y * keb + pl.y);
                    }
                    dq = __ffma2_rn(md, kk, dq);
                    dk = __ffma2_rn(md, q, dk);
                    if (r == Cn - 1) dl = __fadd2_rn(dl, rsum);
                    *reinterpret_cast<uint32_t *>(gdq + o) = pack_bf16(dq.x, dq.y);
                    const float2 dkt = __ffma2_rn(dg, bb, dk), dbt = __fmul2_rn(dg, kk);
                    *reinterpret_cast<uint32_t *>(gdk + o) = pack_bf16(dkt.x, dkt.y);
                    *reinterpret_cast<uint32_t *>(gdb + o) = pack_bf16(dbt.x, dbt.y);
                    dla_r[i] = dl.x;
                    dlb_r[i] = dl.y;
                    psum = __fadd2_rn(psum, dl);
                }
            }
            s_dpart[s2][c2] = psum.x;
            s_dpart[s2][c2 + 1] = psum.y;
            __syncthreads();
            float acca = 0.f, accb = 0.f;
#pragma unroll
            for (int s = 0; s < P2; ++s)
                if (s > s2) { acca += s_dpart[s][c2]; accb += s_dpart[s][c2 + 1]; }
#pragma unroll
            for (int i = RS2 - 1; i >= 0; --i) {
                const int r = s2 * RS2 + i;
                if (r < Cn) {
                    acca += dla_r[i];
                    accb += dlb_r[i];
                    *reinterpret_cast<uint32_t *>(static_cast<bf16 *>(a.dlog_alpha) +
                                                  ((row0 + n * C + r) * H + h) * DK + c2) =
                        pack_bf16(acca, accb);
                }
            }
        }
    }

    // ---- Token-level gradients with four key channels per thread: lane =
    // channel quad, warp = 4-row segment of the chunk (DK = 128, NT = 512), so
    // that every raw-row load and gradient store moves 8 bytes and a warp's
    // store covers 256 contiguous bytes of one token row.
    static constexpr int NQ = DK / 4, P4 = NT / NQ, R4 = C / P4;
    struct RawRows4 {
        uint2 q[R4], k[R4], b[R4], la[R4];
    };
    __device__ void load_rows4(RawRows4 &raw, int n, int Cn) const {
        const int c4 = 4 * (tid % NQ), s4 = tid / NQ;
        const bf16 *gla = static_cast<const bf16 *>(a.log_alpha);
        const unsigned short *sb = reinterpret_cast<const unsigned short *>(gb);
        const unsigned short *sla = reinterpret_cast<const unsigned short *>(gla);
#pragma unroll
        for (int i = 0; i < R4; ++i) {
            const int r = min(s4 * R4 + i, Cn - 1);
            const size_t o = ((row0 + n * C + r) * H + h) * DK + c4;
            const size_t os = (row0 + n * C + r) * H + h;  // a scalar gate's element
            raw.q[i] = *reinterpret_cast<const uint2 *>(gq + o);
            raw.k[i] = *reinterpret_cast<const uint2 *>(gk + o);
            if (GATES == kGatesFull) {
                raw.b[i] = *reinterpret_cast<const uint2 *>(gb + o);
            } else {
                const uint32_t x = sb[os] | ((uint32_t)sb[os] << 16);
                raw.b[i] = make_uint2(x, x);
            }
            if (GATES != kGatesGDN) {
                raw.la[i] = *reinterpret_cast<const uint2 *>(gla + o);
            } else {
                const uint32_t x = sla[os] | ((uint32_t)sla[os] << 16);
                raw.la[i] = make_uint2(x, x);
            }
        }
    }
    // One channel pair of a fast chunk: dq, dk, db before the diagonal-of-M
    // terms, and the dlog_alpha term (run = the in-chunk decay prefix L).
    struct Pair {
        float2 dq, dg, dk, dl;
    };
    static __device__ __forceinline__ Pair fast_pair(float2 dqt, float2 dgt, float2 dkb, float2 q, float2 k, float2 bb,
                                                     float2 run) {
        const float2 e = make_float2(__expf(run.x), __expf(run.y));
        const float2 ie = make_float2(__expf(-run.x), __expf(-run.y));
        Pair p;
        p.dq = __fmul2_rn(dqt, e);
        p.dg = __fmul2_rn(dgt, e);
        p.dk = __fmul2_rn(dkb, ie);
        p.dl = __fmul2_rn(p.dk, make_float2(-k.x, -k.y));
        p.dl = __ffma2_rn(p.dg, __fmul2_rn(bb, k), p.dl);
        p.dl = __ffma2_rn(p.dq, q, p.dl);
        return p;
    }
    // ... and of a slow chunk, from its exact L and the term-by-term Gram
    // gradients PQ, PG, PK, PL (lend = L at the chunk's last token).
    static __device__ __forceinline__ Pair slow_pair(float2 dqt, float2 dgt, float2 dkb, float2 q, float2 k, float2 bb,
                                                     float2 lam, float2 lend, float2 pq, float2 pg, float2 pk,
                                                     float2 pl) {
        const float ea = __expf(lam.x), eb = __expf(lam.y);
        const float kea = __expf(lend.x - lam.x), keb = __expf(lend.y - lam.y);
        Pair p;
        p.dq = make_float2(dqt.x * ea + pq.x, dqt.y * eb + pq.y);
        p.dg = make_float2(dgt.x * ea + pg.x, dgt.y * eb + pg.y);
        p.dk = make_float2(dkb.x * kea + pk.x, dkb.y * keb + pk.y);
        p.dl = make_float2(dqt.x * q.x * ea + dgt.x * bb.x * k.x * ea - dkb.x * k.x * kea + pl.x,
                           dqt.y * q.y * eb + dgt.y * bb.y * k.y * eb - dkb.y * k.y * keb + pl.y);
        return p;
    }
    // dq, dk, db and dlog_alpha from the fp32 staging tiles DQT, DGT, DKB (and
    // PQ.. for a slow chunk).  seg: [P4][DK] sums of log_alpha over the rows
    // before each 4-row segment (a fast chunk's decay prefix); dseg: a free [P4][DK] fp32 area
    // for the segment sums of dL.  All of seg, dseg and s_rs 16-byte aligned.
    // rows_done() runs on every thread once all threads have read the staging
    // tiles and s_rs (after a barrier).
    template <class F>
    __device__ void token_grads4(int n, int Cn, bool slow, const RawRows4 &raw, const float (*seg)[DK],
                                 float (*dseg)[DK], F &&rows_done) {
        const int c4 = 4 * (tid % NQ), s4 = tid / NQ;
        const float4 lend4 = slow ? *reinterpret_cast<const float4 *>(LAM + (Cn - 1) * DK + c4)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
        float4 rsum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < NRS; ++i) {
            const float4 t = *reinterpret_cast<const float4 *>(&s_rs[i][c4]);
            rsum.x += t.x; rsum.y += t.y; rsum.z += t.z; rsum.w += t.w;
        }
        // in-chunk decay prefix at the start of this thread's segment
        const float4 pre = *reinterpret_cast<const float4 *>(&seg[s4][c4]);
        float2 run0 = make_float2(pre.x, pre.y), run1 = make_float2(pre.z, pre.w);
        bf16 *__restrict__ gdq = static_cast<bf16 *>(a.dq);
        bf16 *__restrict__ gdk = static_cast<bf16 *>(a.dk);
        bf16 *__restrict__ gdb = static_cast<bf16 *>(a.db);
        float2 dl0[R4], dl1[R4];
        float2 ps0 = make_float2(0.f, 0.f), ps1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < R4; ++i) {
            const int r = s4 * R4 + i;
            dl0[i] = make_float2(0.f, 0.f);
            dl1[i] = make_float2(0.f, 0.f);
            if (r < Cn) {
                const size_t o = ((row0 + n * C + r) * H + h) * DK + c4;
                const float2 q0 = unpack_bf16(raw.q[i].x), q1 = unpack_bf16(raw.q[i].y);
                const float2 k0 = unpack_bf16(raw.k[i].x), k1 = unpack_bf16(raw.k[i].y);
                const float2 b0 = unpack_bf16(raw.b[i].x), b1 = unpack_bf16(raw.b[i].y);
                const float4 dqt = *reinterpret_cast<const float4 *>(DQT + stg<DK>(r, c4));
                const float4 dgt = *reinterpret_cast<const float4 *>(DGT + stg<DK>(r, c4));
                const float4 dkb = *reinterpret_cast<const float4 *>(DKB + stg<DK>(r, c4));
                Pair p0, p1;
                if (!slow) {
                    run0 = __fadd2_rn(run0, unpack_bf16(raw.la[i].x));
                    run1 = __fadd2_rn(run1, unpack_bf16(raw.la[i].y));
                    p0 = fast_pair(make_float2(dqt.x, dqt.y), make_float2(dgt.x, dgt.y), make_float2(dkb.x, dkb.y),
                                   q0, k0, b0, run0);
                    p1 = fast_pair(make_float2(dqt.z, dqt.w), make_float2(dgt.z, dgt.w), make_float2(dkb.z, dkb.w),
                                   q1, k1, b1, run1);
                } else {
                    const float4 lam = *reinterpret_cast<const float4 *>(LAM + r * DK + c4);
                    const float4 pq = *reinterpret_cast<const float4 *>(PQ + r * DK + c4);
                    const float4 pg = *reinterpret_cast<const float4 *>(PG + r * DK + c4);
                    const float4 pk = *reinterpret_cast<const float4 *>(PK + r * DK + c4);
                    const float4 pl = *reinterpret_cast<const float4 *>(PL + r * DK + c4);
                    p0 = slow_pair(make_float2(dqt.x, dqt.y), make_float2(dgt.x, dgt.y), make_float2(dkb.x, dkb.y),
                                   q0, k0, b0, make_float2(lam.x, lam.y), make_float2(lend4.x, lend4.y),
                                   make_float2(pq.x, pq.y), make_float2(pg.x, pg.y), make_float2(pk.x, pk.y),
                                   make_float2(pl.x, pl.y));
                    p1 = slow_pair(make_float2(dqt.z, dqt.w), make_float2(dgt.z, dgt.w), make_float2(dkb.z, dkb.w),
                                   q1, k1, b1, make_float2(lam.z, lam.w), make_float2(lend4.z, lend4.w),
                                   make_float2(pq.z, pq.w), make_float2(pg.z, pg.w), make_float2(pk.z, pk.w),
                                   make_float2(pl.z, pl.w));
                }
                // the diagonal of M carries no decay: its gradient s_dmd goes to dq and dk directly
                const float2 md = make_float2(s_dmd[r], s_dmd[r]);
                p0.dq = __ffma2_rn(md, k0, p0.dq);
                p1.dq = __ffma2_rn(md, k1, p1.dq);
                p0.dk = __ffma2_rn(md, q0, p0.dk);
                p1.dk = __ffma2_rn(md, q1, p1.dk);
                if (r == Cn - 1) {
                    p0.dl = __fadd2_rn(p0.dl, make_float2(rsum.x, rsum.y));
                    p1.dl = __fadd2_rn(p1.dl, make_float2(rsum.z, rsum.w));
                }
                const float2 dk0 = __ffma2_rn(p0.dg, b0, p0.dk), dk1 = __ffma2_rn(p1.dg, b1, p1.dk);
                const float2 db0 = __fmul2_rn(p0.dg, k0), db1 = __fmul2_rn(p1.dg, k1);
                *reinterpret_cast<uint2 *>(gdq + o) = make_uint2(pack_bf16(p0.dq.x, p0.dq.y), pack_bf16(p1.dq.x, p1.dq.y));
                *reinterpret_cast<uint2 *>(gdk + o) = make_uint2(pack_bf16(dk0.x, dk0.y), pack_bf16(dk1.x, dk1.y));
                if (GATES == kGatesFull) {
                    *reinterpret_cast<uint2 *>(gdb + o) =
                        make_uint2(pack_bf16(db0.x, db0.y), pack_bf16(db1.x, db1.y));
                } else {  // dbeta = sum over the key channels of db, plus that of dw
                    const float sdb = warp_sum(db0.x + db0.y + db1.x + db1.y);
                    if (lane == 0) gdb[(row0 + n * C + r) * H + h] = __float2bfloat16_rn(sdb + s_dbw[r]);
                }
                dl0[i] = p0.dl;
                dl1[i] = p1.dl;
                ps0 = __fadd2_rn(ps0, p0.dl);
                ps1 = __fadd2_rn(ps1, p1.dl);
            }
        }
        // in-chunk reverse cumulative sum of dL: the later segments, then this
        // thread's rows from the last up
        *reinterpret_cast<float4 *>(&dseg[s4][c4]) = make_float4(ps0.x, ps0.y, ps1.x, ps1.y);
        __syncthreads();
        rows_done();
        float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll 4
        for (int s = s4 + 1; s < P4; ++s) {
            const float4 t = *reinterpret_cast<const float4 *>(&dseg[s][c4]);
            acc0 = __fadd2_rn(acc0, make_float2(t.x, t.y));
            acc1 = __fadd2_rn(acc1, make_float2(t.z, t.w));
        }
        bf16 *__restrict__ gdl = static_cast<bf16 *>(a.dlog_alpha);
#pragma unroll
        for (int i = R4 - 1; i >= 0; --i) {
            const int r = s4 * R4 + i;
            if (r < Cn) {
                acc0 = __fadd2_rn(acc0, dl0[i]);
                acc1 = __fadd2_rn(acc1, dl1[i]);
                if (GATES != kGatesGDN) {
                    *reinterpret_cast<uint2 *>(gdl + ((row0 + n * C + r) * H + h) * DK + c4) =
                        make_uint2(pack_bf16(acc0.x, acc0.y), pack_bf16(acc1.x, acc1.y));
                } else {  // a scalar decay: the sum over the key channels
                    const float sdl = warp_sum(acc0.x + acc0.y + acc1.x + acc1.y);
                    if (lane == 0) gdl[(row0 + n * C + r) * H + h] = __float2bfloat16_rn(sdl);
                }
            }
        }
    }
};

}  // namespace cbwd
}  // namespace gdn2
