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
#include "chunk_common.cuh"
#include "gdn2.h"
#include "launch.h"

namespace gdn2 {
namespace cfwd {

using namespace chunk;

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
__device__ __forceinline__ ChunkTiles stage_tiles(unsigned char *smem, int s) {
    using L = Smem<DK, DV>;
    unsigned char *p = smem + s * L::STAGE;
    return {reinterpret_cast<bf16 *>(p + L::OQ), reinterpret_cast<bf16 *>(p + L::OK),
            reinterpret_cast<bf16 *>(p + L::OLA), reinterpret_cast<bf16 *>(p + L::OB),
            reinterpret_cast<bf16 *>(p + L::OV), reinterpret_cast<bf16 *>(p + L::OW)};
}

template <int DK, int DV>
__device__ __forceinline__ void issue_chunk(const ChunkFwdArgs &a, ChunkTiles st, const SeqView &sv, int h, int n) {
    load_token_tile<DK>(st.q, static_cast<const bf16 *>(a.q), sv.row0, sv.len, h, n, a.H);
    load_token_tile<DK>(st.k, static_cast<const bf16 *>(a.k), sv.row0, sv.len, h, n, a.H);
    load_token_tile<DK>(st.la, static_cast<const bf16 *>(a.log_alpha), sv.row0, sv.len, h, n, a.H);
    load_token_tile<DK>(st.b, static_cast<const bf16 *>(a.b), sv.row0, sv.len, h, n, a.H);
    if (!a.transition) {  // (a transition pass has no write term: its v and w tiles are zeroed instead)
        load_token_tile<DV>(st.v, static_cast<const bf16 *>(a.v), sv.row0, sv.len, h, n, a.H);
        load_token_tile<DV>(st.w, static_cast<const bf16 *>(a.w), sv.row0, sv.len, h, n, a.H);
    }
    cp_commit();
}

// One CTA per (batch, head).  With a.states set (the backward's state pass)
// the bf16 state at every chunk boundary is written to
// a.states[bh][n][DK][DV] (n = 0..nchunks) and o may be null.
template <int DK, int DV>
__global__ void __launch_bounds__(NTHR, 1) chunk_fwd_kernel(ChunkFwdArgs a) {
    using L = Smem<DK, DV>;
    constexpr int WR = DK / 4, WC = DV / 2;  // state tile of a warp
    constexpr int MTS = WR / 16, NTS = WC / 8;
    constexpr int NTV = DV / 8, NTK = DK / 8;

    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ IntraShared<DK> sh;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
    const SeqView sv = seq_view(a.cu_seqlens, b, h, a.B, a.T, a.H);
    if (!sv.ok) {  // packed-sequence offsets out of range: nothing of this sequence is touched
        if (tid == 0) record_status(a.status, GDN2_ERR_INVALID_ARG);
        return;
    }
    const int nchunks = sv.nchunks;
    bf16 *S16 = reinterpret_cast<bf16 *>(smem + L::OS16);
    float *lam_ws = a.ws ? a.ws + (size_t)bh * a.ws_stride : nullptr;
    const bool with_o = a.o != nullptr;
    auto keep_tile = [&](int n) {
        return static_cast<unsigned char *>(a.intra) + (sv.cslot + n) * intra_tile_bytes(DV);
    };

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
                S[mt][nt][e] = a.transition ? (c == j ? 1.f : 0.f)
                               : (a.S0 ? a.S0[(size_t)bh * DK * DV + (size_t)c * DV + j] : 0.f);
            }
    // bf16 copy of the state into shared memory (and to a.states[n] when set)
    auto write_S16 = [&](int n) {
        bf16 *gs = a.states ? static_cast<bf16 *>(a.states) + (sv.sslot + n) * DK * DV : nullptr;
#pragma unroll
        for (int mt = 0; mt < MTS; ++mt)
#pragma unroll
            for (int nt = 0; nt < NTS; ++nt) {
                const int c = c0 + 16 * mt + (lane >> 2);
                const int j = j0 + 8 * nt + 2 * (lane & 3);
                const uint32_t lo = pack_bf16(S[mt][nt][0], S[mt][nt][1]);
                const uint32_t hi = pack_bf16(S[mt][nt][2], S[mt][nt][3]);
                *reinterpret_cast<uint32_t *>(S16 + swz<DV, DK>(c, j)) = lo;
                *reinterpret_cast<uint32_t *>(S16 + swz<DV, DK>(c + 8, j)) = hi;
                if (gs) {
                    *reinterpret_cast<uint32_t *>(gs + (size_t)c * DV + j) = lo;
                    *reinterpret_cast<uint32_t *>(gs + (size_t)(c + 8) * DV + j) = hi;
                }
            }
    };
    write_S16(0);

    if (nchunks > 0) issue_chunk<DK, DV>(a, stage_tiles<DK, DV>(smem, 0), sv, h, 0);
    else cp_commit();
    if (nchunks > 1) issue_chunk<DK, DV>(a, stage_tiles<DK, DV>(smem, 1), sv, h, 1);
    else cp_commit();

    for (int n = 0; n < nchunks; ++n) {
        const int stg = n & 1;
        ChunkTiles st = stage_tiles<DK, DV>(smem, stg);
        float *A32 = reinterpret_cast<float *>(L::REUSE ? reinterpret_cast<unsigned char *>(st.k)
                                                         : smem + L::ODED);
        float *T32 = reinterpret_cast<float *>(L::REUSE ? reinterpret_cast<unsigned char *>(st.w)
                                                         : smem + L::ODED + L::REG);
        bf16 *W16 = reinterpret_cast<bf16 *>(A32);                 // after the solve
        bf16 *T16 = reinterpret_cast<bf16 *>(T32);                 // [64][64]
        bf16 *M16 = reinterpret_cast<bf16 *>(T32) + C * C;         // [64][64]
        bf16 *U16 = st.v;                                          // after W, Uv

        cp_wait<1>();
        __syncthreads();
        if (a.transition) {  // no write term: w . v = 0 (the slots hold other tiles' data otherwise)
            for (int id = threadIdx.x; id < 2 * C * DV / 8; id += NTHR)
                reinterpret_cast<uint4 *>(id < C * DV / 8 ? st.v : st.w)[id % (C * DV / 8)] = make_uint4(0, 0, 0, 0);
            __syncthreads();
        }
        const bool slow = intra_chunk<DK, DV>(st, A32, T32, view(sh), lam_ws, false);
        // T and M (then U, below) for the backward, as their shared-memory images
        if (a.intra) copy_smem_to_global(keep_tile(n), T16, 2 * C * C * 2);

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
            warp_gemm<1, NTV, true, false, DK, DV, C, DK>(accV, W16, 16 * warp, S16, 0, DK, lane);
            store_tile_bf16<NTV, DV>(accV, U16, 16 * warp, lane, 1.f);
        } else if (with_o) {
            warp_gemm<1, NTV, true, false, DK, DV, C, DK>(accV, st.q, 16 * (warp & 3), S16, 0, DK, lane);
        }
        __syncthreads();

        if (a.intra) copy_smem_to_global(keep_tile(n) + 2 * C * C * 2, U16, C * DV * 2);
        // ---- O += M U, store o
        if (warp >= 4 && with_o) {
            warp_gemm<1, NTV, true, false, 64, DV>(accV, M16, 16 * (warp & 3), U16, 0, C, lane);
            const int rl = 16 * (warp & 3) + (lane >> 2);
            bf16 *o = static_cast<bf16 *>(a.o);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int t = n * C + rl + 8 * half;
                if (t < sv.len) {
                    bf16 *orow = o + ((sv.row0 + t) * a.H + h) * DV;
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
                const float g0 = sh.gamma[c0 + 16 * mt + (lane >> 2)], g1 = sh.gamma[c0 + 16 * mt + (lane >> 2) + 8];
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
                const float g0 = sh.gamma[c0 + 16 * mt + (lane >> 2)], g1 = sh.gamma[c0 + 16 * mt + (lane >> 2) + 8];
#pragma unroll
                for (int nt = 0; nt < NTS; ++nt) {
                    S[mt][nt][0] *= g0; S[mt][nt][1] *= g0; S[mt][nt][2] *= g1; S[mt][nt][3] *= g1;
                }
            }
        }
        write_S16(n + 1);
        __syncthreads();
        if (n + 2 < nchunks) issue_chunk<DK, DV>(a, st, sv, h, n + 2);
        else cp_commit();
    }
    cp_wait<0>();

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
    if (dk == 128 && dv == 128) return launch_chunk_fwd_tc(a, s);
    if (dk == 128 && dv == 64) return cfwd::launch_t<128, 64>(a, s);
    if (dk == 64 && dv == 128) return cfwd::launch_t<64, 128>(a, s);
    return cfwd::launch_t<64, 64>(a, s);
}

size_t chunk_fwd_ws_bytes(int B, int H, int dk) { return (size_t)B * H * chunk::C * dk * sizeof(float); }

}  // namespace gdn2
