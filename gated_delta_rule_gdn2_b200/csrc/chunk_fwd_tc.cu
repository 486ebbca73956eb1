// Chunk-parallel forward for dk = dv = 128 with every chunk product on the
// fifth-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// Same algebra as chunk_fwd.cu ("Why NVIDIA Gated DeltaNet-2 separates erase
// and write gates", section "Gated Delta Rule-2: per-channel erase/write
// split"; WY form from the laonpeople Gated DeltaNet page): per chunk
//   A = Gt Kb^T, M = Qt Kb^T,  T = (I + A)^{-1},
//   U = T (w . v) - (T Gt) S,   O = Qt S + M U,   S <- Diag(gam) (S + Kb^T U).
// The fp32 state S lives in TMEM (128 lanes = key channels x 128 columns)
// for the whole sequence.  Two warp groups of 8 warps share the work: group
// A forms chunk m's decay prefix and operands Qt, Gt, Kb and w . v, issues the
// two Grams (M = N = 64, K = 128), reads back A (fp32, for the WY solve) and
// M (bf16) and inverts A's four 16x16 diagonal blocks; group B runs chunk
// m - 1's state chain: the rest of the WY solve (TF32 tensor-core levels on
// the diagonal-block inverses, chunk_common.cuh), then
//   T Gt (M = 64, N = 128, K = 64, into O's columns) and T (w . v), which
//   need no state;
//   U += (-W) S (K = 128, bf16 S copy in shared memory as B), then O = Qt S,
//   so that U, which the chain waits for, completes first;
//   O += M U (committed first: the O epilogue runs under the next one) and
//   S += Kb^T U (M = 128),
// reading results back with the 16x256b TMEM load shape (the register layout
// of a warp-level m16n8 fragment) to form -W and U in bf16.  S is scaled by
// gam in TMEM (32x32b load/store) and copied to bf16 for the next chunk.  A
// chunk whose decay spans more than e^{-64} takes its Grams term by term in
// fp32 inside the shared intra-chunk stage (group A, with its own solve).
// Tiles arrive by TMA into two stages, the pipeline's buffers; the tiles kept
// for the backward leave as bulk stores and O as a TMA tensor store of its
// bf16 image.  Every wait on an mbarrier is bounded: on expiry the kernel
// records GDN2_ERR_TIMEOUT in the device status word, frees its tensor memory
// and returns.
#include "chunk_common.cuh"
#include "gdn2.h"
#include "launch.h"
#include "tc_tiles.cuh"
#include "tma_host.h"

namespace gdn2 {
namespace cfwd_tc {

using namespace chunk;

constexpr int D = 128;
constexpr int TILE = C * D * 2;          // one [64][128] bf16 tile: 16 KB
constexpr int STAGE = 6 * TILE;          // q k log_alpha b v w
constexpr int OS16 = 2 * STAGE;          // bf16 copy of S: [2 col blocks][128 rows][64]
constexpr int OSMALL = OS16 + D * D * 2;

// Two warp groups of 256 threads: A (warps 0..7) runs the intra-chunk stage
// of chunk m while B (warps 8..15) runs the state chain of chunk m - 1; the
// two stages of input tiles are the pipeline's buffers.
constexpr int NT = 512, NG = 256;
using GA = Grp<1, NG, 0>;
using GB = Grp<2, NG, NG>;

struct Small {
    float part[NG / (D / 2) - 1][D];  // group A: segment sums of log_alpha
    float gamma[2][D];    // per stage: gam = e^{L_end} of its chunk
    int slow[2];          // per stage: the chunk took the exact path
    uint64_t mbar_a;      // MMA completion, group A
    uint64_t mbar_b;      // MMA completion, group B
    uint64_t mbar_o;      // MMA completion, group B's O products (a second barrier: each keeps one phase in flight)
    uint64_t mbar_ld[2];  // tile loads of stage 0 and 1
    uint64_t ready[2];    // stage s: its intra-chunk stage is done
    uint64_t mbar_fin[2]; // the issuing threads' last tensor-core work (groups A, B), at the end
    uint64_t mbar_g;      // the fused epilogue's output-gate tile
    int ld_issued[2];     // per stage: tile loads issued (thread tb = 0) ...
    int ld_waited[2];     // ... and waited for (group A)
    int g_issued, g_landed;  // output-gate tiles issued and landed (group B)
    uint32_t tmem;
    int abort;
};
constexpr int BYTES = OSMALL + (int)sizeof(Small);
static_assert(BYTES <= 232448, "shared memory per block");

// Tensor memory: group B's U (T Gt, then T (w . v) + (-W) S), O (Qt S, then
// + M U) and the state S (fp32, 128 key rows x 128 value columns); group A's
// Grams (A | M, 64 columns each).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t COL_U = 0, COL_O = 128, COL_S = 256, COL_G = 384;
constexpr uint32_t ID64x64_K_K = tc::idesc_bf16(64, 64, false, false);
constexpr uint32_t ID64x128_K_MN = tc::idesc_bf16(64, 128, false, true);
constexpr uint32_t IDESC_S = tc::idesc_bf16(128, 128, true, true);  // A, B MN-major

using tct::Frag;
using tct::ld_frag;
using tct::mma_tiles;
using tct::store_frag_bf16;

__device__ __forceinline__ ChunkTiles stage_tiles(unsigned char *smem, int s) {
    unsigned char *p = smem + s * STAGE;
    return {reinterpret_cast<bf16 *>(p), reinterpret_cast<bf16 *>(p + TILE), reinterpret_cast<bf16 *>(p + 2 * TILE),
            reinterpret_cast<bf16 *>(p + 3 * TILE), reinterpret_cast<bf16 *>(p + 4 * TILE),
            reinterpret_cast<bf16 *>(p + 5 * TILE)};
}

// TMA tensor maps of the six token tensors (whole-tile boxes, token_tile_map)
// and of the output o (64 x 64 boxes).
struct FwdMaps {
    CUtensorMap q, k, la, b, v, w, o, g;  // g: the output gate of the fused epilogue
    CUtensorMap qphi;                     // segments: the transition pass's rows Phi_t^T q_t
};

// Chunk n's six token tiles into a stage (one thread; one box per tile),
// completion counted in bytes on the stage's mbarrier.  Rows past the end of
// the tensor read as zeros.
// With scalar gates (KDA / GDN) the b and w tiles (and, for GDN, the
// log_alpha tile) are not loaded: expand_gates fills them from the scalars.
// A transition pass (no_vw) reads no v and w either.
__device__ __forceinline__ void issue_chunk(const FwdMaps &m, ChunkTiles st, const SeqView &sv, int h, int n,
                                            uint64_t *mbar, int gates, bool no_vw = false) {
    const int ntiles = no_vw ? 4 : (gates == kGatesFull ? 6 : (gates == kGatesKDA ? 4 : 3));
    tc::mbar_expect_tx(mbar, ntiles * TILE);
    const int t = sv.map_t0 + n * C, b = sv.map_b;
    if (gates != kGatesGDN) tc::tma_load_5d(st.la, &m.la, 0, t, 0, h, b, mbar);
    tc::tma_load_5d(st.q, &m.q, 0, t, 0, h, b, mbar);
    tc::tma_load_5d(st.k, &m.k, 0, t, 0, h, b, mbar);
    if (no_vw || gates == kGatesFull) tc::tma_load_5d(st.b, &m.b, 0, t, 0, h, b, mbar);
    if (!no_vw) tc::tma_load_5d(st.v, &m.v, 0, t, 0, h, b, mbar);
    if (!no_vw && gates == kGatesFull) tc::tma_load_5d(st.w, &m.w, 0, t, 0, h, b, mbar);
}

// Scalar gates into whole tiles: row r of the b and w tiles (and, for GDN, of
// the log_alpha tile) holds the scalar of token n*C + r in every column; rows
// past the sequence's end hold zeros (a zero token).  The NTG threads of G.
template <class G, int NTG, int GATES>
__device__ __forceinline__ void expand_gates(ChunkTiles st, const ChunkFwdArgs &a, const SeqView &sv, int h, int n) {
    constexpr int ntiles = GATES == kGatesGDN ? 3 : 2;
    const int valid = min(C, sv.len - n * C);
    const unsigned short *beta = static_cast<const unsigned short *>(a.b);
    const unsigned short *lsc = static_cast<const unsigned short *>(a.log_alpha);
    for (int id = G::tid(); id < ntiles * 2 * C * 8; id += NTG) {
        const int t = id / (2 * C * 8), rem = id % (2 * C * 8);
        const int blk = rem / (C * 8), r = (rem % (C * 8)) / 8, ch = rem % 8;
        uint32_t x = 0;
        if (r < valid) {
            const size_t o = (sv.row0 + (size_t)n * C + r) * a.H + h;
            x = t < 2 ? beta[o] : lsc[o];
        }
        x |= x << 16;
        bf16 *tile = t == 0 ? st.b : (t == 1 ? st.w : st.la);
        *reinterpret_cast<uint4 *>(tile + blk * (C * 64) + r * 64 + ch * 8) = make_uint4(x, x, x, x);
    }
}

// Rows Cn .. 63 of the six tiles of a stage to zero (the last chunk of a
// packed sequence, whose box reaches into the next sequence): zero tokens
// leave the state and the other rows unchanged.  The NT threads of G.
template <class G, int NTG>
__device__ __forceinline__ void zero_tail_rows(ChunkTiles st, int Cn) {
    const int rows = C - Cn;  // (the six tiles lie back to back from st.q, TILE bytes each)
    for (int id = G::tid(); id < 6 * 2 * rows * 8; id += NTG) {
        const int t = id / (2 * rows * 8), rem = id % (2 * rows * 8);
        const int blk = rem / (rows * 8), r = Cn + (rem % (rows * 8)) / 8, ch = rem % 8;
        *reinterpret_cast<uint4 *>(st.q + t * (C * D) + blk * (C * 64) + r * 64 + ch * 8) = make_uint4(0u, 0u, 0u, 0u);
    }
}

// Compile-time forms: GATES (the gate form) and MODE (kPlain, kSegments: the
// segment path's local and transition passes, kGated: the output epilogue in
// the O epilogue), so that the plain form carries no branch on them.
constexpr int kPlain = 0, kSegments = 1, kGated = 2;
template <int GATES, int MODE>
__global__ void __launch_bounds__(NT, 1) chunk_fwd_tc_kernel(ChunkFwdArgs a, const __grid_constant__ FwdMaps maps) {
    extern __shared__ __align__(1024) unsigned char smem[];
    Small &sm = *reinterpret_cast<Small *>(smem + OSMALL);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tc::smem_addr(smem) & 1023u) {  // the operand atoms need 1 KB alignment
        if (tid == 0) record_status(a.status, GDN2_ERR_CUDA);
        return;
    }
    int b, h;
    SeqView sv;
    bool phi = false;  // a segment's transition pass
    const float *S0p;  // this CTA's start state (nullptr: zero; a transition pass starts from I)
    float *STp;        // and its end state (or nullptr)
    void *op = a.o;    // its output rows
    if constexpr (MODE != kSegments) {
        const int bh = blockIdx.x;
        b = bh / a.H;
        h = bh % a.H;
        sv = seq_view(a.cu_seqlens, b, h, a.B, a.T, a.H);
        S0p = a.S0 ? a.S0 + (size_t)bh * D * D : nullptr;
        STp = a.S_T ? a.S_T + (size_t)bh * D * D : nullptr;
    } else {
        const int P = a.seg_P, nloc = a.B * P * a.H;
        int i = blockIdx.x, p;
        phi = i >= nloc;
        if (phi) i -= nloc;
        h = i % a.H;
        const int bp = i / a.H;
        b = phi ? bp / (P - 1) : bp / P;
        p = phi ? bp % (P - 1) + 1 : bp % P;
        const int nch = a.T / C, base = nch / P, rem = nch % P;
        const int c0 = p * base + min(p, rem), cn = base + (p < rem ? 1 : 0);
        sv.row0 = (size_t)b * a.T + (size_t)c0 * C;
        sv.len = cn * C;
        sv.nchunks = cn;
        sv.cslot = sv.sslot = 0;
        sv.map_b = b;
        sv.map_t0 = c0 * C;
        sv.ok = true;
        S0p = (!phi && p == 0 && a.S0) ? a.S0 + ((size_t)b * a.H + h) * D * D : nullptr;
        STp = (phi ? a.seg_phi : a.seg_loc) + (size_t)i * D * D;
        if (phi) op = a.seg_qphi;
    }
    if (!sv.ok) {  // packed-sequence offsets out of range: nothing of this sequence is touched
        if (tid == 0) record_status(a.status, GDN2_ERR_INVALID_ARG);
        return;
    }
    const int nchunks = sv.nchunks;
    const bool packed = a.cu_seqlens != nullptr;

    if (warp == 0) tc::tmem_alloc(&sm.tmem, kTmemCols);
    if (tid == 0) {
        tc::mbar_init(&sm.mbar_a, 1);
        tc::mbar_init(&sm.mbar_b, 1);
        tc::mbar_init(&sm.mbar_o, 1);
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(&sm.mbar_ld[i], 1);
            tc::mbar_init(&sm.ready[i], 1);
            tc::mbar_init(&sm.mbar_fin[i], 1);
            sm.ld_issued[i] = 0;
            sm.ld_waited[i] = 0;
        }
        tc::mbar_init(&sm.mbar_g, 1);
        sm.g_issued = 0;
        sm.g_landed = 0;
        tc::fence_mbar_init();
        sm.abort = 0;
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = sm.tmem;
    // TMEM sub-partition of this warp: its 32 lanes (state rows 32 p ..) and
    // the rows 16 p .. 16 p + 15 of a 64-row product; two warps of each group
    // share a sub-partition and take the column halves hc = 0, 1.
    const int p = warp & 3, hc = (warp >> 2) & 1;
    const uint32_t lane_base = (uint32_t)(32 * p) << 16;
    // Bounded wait on an mbarrier phase; a timeout is recorded and ends the pass.
    const uint32_t wait_limit = a.wait_limit ? a.wait_limit : tc::kWaitLimit;
    auto wait_on = [&](uint64_t *mbar, uint32_t &phase) {
        const bool ok = tc::mbar_wait(mbar, phase, wait_limit);
        if (!ok) {
            sm.abort = 1;
            record_status(a.status, GDN2_ERR_TIMEOUT);
        }
        phase ^= 1;
        tc::fence_after();
        return ok;
    };
    // ... on the barrier of stage s, whose phase is bit s of a per-thread word
    // (a phase array indexed by the stage would live in local memory)
    auto wait_stage = [&](uint64_t *mbar, uint32_t &bits, int s) {
        uint32_t ph = (bits >> s) & 1u;
        bits ^= 1u << s;
        return wait_on(mbar, ph);
    };

    if (warp < 8) {
        // ================= group A: decay prep, Grams, A and M =================
        // (a fast chunk's WY solve runs in group B; a slow chunk takes its Grams
        // term by term and its solve in the intra-chunk stage here)
        float *lam_ws = a.ws ? a.ws + (size_t)blockIdx.x * a.ws_stride : nullptr;
        uint32_t ph_a = 0, ph_ld = 0;
        for (int m = 0; m < nchunks; ++m) {
            const int s = m & 1;
            ChunkTiles st = stage_tiles(smem, s);
            float *A32 = reinterpret_cast<float *>(st.k);  // k and w slots are free after the prep
            float *T32 = reinterpret_cast<float *>(st.w);
            bf16 *M16 = reinterpret_cast<bf16 *>(T32) + C * C;

            if (wait_stage(&sm.mbar_ld[s], ph_ld, s) && tid == 0) ++sm.ld_waited[s];  // (landed)
            GA::sync();
            if (sm.abort) break;
            if (packed && sv.len - m * C < C) {
                zero_tail_rows<GA, NG>(st, sv.len - m * C);
                GA::sync();
            }
            if constexpr (GATES != kGatesFull) {
                expand_gates<GA, NG, GATES>(st, a, sv, h, m);
                GA::sync();
            }
            if (phi) {  // a transition pass: no write term (w . v = 0)
                for (int id = tid; id < 2 * C * D / 8; id += NG)
                    reinterpret_cast<uint4 *>(id < C * D / 8 ? st.v : st.w)[id % (C * D / 8)] = make_uint4(0, 0, 0, 0);
                GA::sync();
            }
            const IntraView<D> iv{sm.part, sm.gamma[s], &sm.slow[s]};
            // a slow chunk takes its Grams term by term, its WY solve and w . v in
            // here; a fast chunk forms w . v below, while its Grams run
            const bool slow = intra_chunk<D, D, NG, GA>(st, A32, T32, iv, lam_ws, false, false, /*grams_ext=*/true,
                                                        /*wv_here=*/false);
            if (!slow) {
                // ---- Grams on the tensor cores: A = Gt Kb^T, M = Qt Kb^T (M = N = 64, K = 128)
                tc::fence_async_smem();
                tc::fence_before();
                GA::sync();
                tc::fence_after();
                if (tid == 0) {
                    mma_tiles<true, true>(tmem + COL_G, st.b, 64, st.la, 64, 8, ID64x64_K_K, false);
                    mma_tiles<true, true>(tmem + COL_G + 64, st.q, 64, st.la, 64, 8, ID64x64_K_K, false);
                    tc::commit(&sm.mbar_a);
                }
                form_wv<D, NG, GA>(st);  // while the tensor cores run
                wait_on(&sm.mbar_a, ph_a);
                {  // A (strictly lower) -> fp32 for the solve
                    Frag<4> f;
                    ld_frag(tmem + lane_base + COL_G + 32 * hc, f);
                    tc::wait_ld();
                    const int r0 = 16 * p + (lane >> 2);
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2) {
                            const int r = r0 + 8 * h2, i = 32 * hc + 8 * nt + 2 * (lane & 3);
                            *reinterpret_cast<float2 *>(A32 + fsw(r, i)) = make_float2(
                                i < r ? f[0][nt][2 * h2] : 0.f, i + 1 < r ? f[0][nt][2 * h2 + 1] : 0.f);
                        }
                }
                GA::sync();  // every thread is done reading w for w . v; A is complete
                // the WY solve's diagonal-block inverses (fp32, in the w tile's first
                // half, which B's T16 takes only after reading them)
                wy_diag<GA>(A32, reinterpret_cast<float *>(st.w));
                {  // M (lower with the diagonal) -> bf16 in the second half of the w tile
                    Frag<4> f;
                    ld_frag(tmem + lane_base + COL_G + 64 + 32 * hc, f);
                    tc::wait_ld();
                    const int r0 = 16 * p + (lane >> 2);
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int r = r0 + (e >> 1) * 8, i = 32 * hc + 8 * nt + 2 * (lane & 3) + (e & 1);
                            if (i > r) f[0][nt][e] = 0.f;
                        }
                    store_frag_bf16<64, 4>(f, M16, 16 * p, 32 * hc, lane, 1.f);
                }
            }
            // hand the stage to group B: every write of it fenced against the
            // tensor cores and the TMA, then one arrival
            tc::fence_async_smem();
            tc::fence_before();
            GA::sync();
            if (tid == 0 && m != a.withhold_ready) tc::mbar_arrive(&sm.ready[s]);
        }
    } else {
        // ================= group B: the state chain =================
        const int tb = tid - NG;
        const bool with_o = op != nullptr;
        const CUtensorMap *omap = phi ? &maps.qphi : &maps.o;
        // The S16 area is free from U's completion to the next chunk's state
        // copy: the chunk's O image goes out from its first half (so that the
        // stage can be refilled without waiting for that store), and the fused
        // output epilogue's gate tile lands in its second half.
        constexpr bool gated = MODE == kGated;  // (with_o: the launch checks o)
        bf16 *S16 = reinterpret_cast<bf16 *>(smem + OS16);
        bf16 *O16 = S16;
        bf16 *G16 = reinterpret_cast<bf16 *>(smem + OS16 + TILE);
        uint32_t ph_g = 0;
        const int c = 32 * p + lane;  // this thread's state row; columns 64 hc .. 64 hc + 63
        const uint32_t t_row = tmem + lane_base + COL_S + 64 * hc;
        auto keep_tile = [&](int n) {
            return static_cast<unsigned char *>(a.intra) + (sv.cslot + n) * intra_tile_bytes(D);
        };
        // the chunk-boundary state n (when requested) as the image of S16 (thread tb = 0)
        auto keep_state = [&](int n) {
            if (a.states) {
                tc::bulk_store(static_cast<bf16 *>(a.states) + (sv.sslot + n) * D * D, S16,
                               D * D * 2);
                tc::bulk_commit();
            }
        };
        // 32 state values of this thread (half i of its 64 columns) <-> TMEM, and
        // their bf16 copy into S16
        auto load_half = [&](int i, float (&v)[32]) {
            tc::ld_32x32b_x32(t_row + 32 * i, v);
            tc::wait_ld();
        };
        auto store_half = [&](int i, const float (&v)[32]) {
            tc::st_32x32b_x32(t_row + 32 * i, v);
            tc::wait_st();
        };
        auto put_half = [&](int i, const float (&v)[32]) {
            bf16 *row = S16 + hc * (D * 64) + c * 64;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint4 u;
                u.x = pack_bf16(v[8 * j + 0], v[8 * j + 1]);
                u.y = pack_bf16(v[8 * j + 2], v[8 * j + 3]);
                u.z = pack_bf16(v[8 * j + 4], v[8 * j + 5]);
                u.w = pack_bf16(v[8 * j + 6], v[8 * j + 7]);
                *reinterpret_cast<uint4 *>(row + (((4 * i + j) ^ (c & 7)) << 3)) = u;
            }
        };
        auto handoff = [&]() {
            tc::fence_async_smem();
            tc::fence_before();
            GB::sync();
            tc::fence_after();
        };

        // initial state into TMEM (its bf16 copy is formed in the first chunk)
        for (int i = 0; i < 2; ++i) {
            float v[32];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float4 x = S0p ? reinterpret_cast<const float4 *>(S0p + (size_t)c * D + 64 * hc + 32 * i)[j]
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
                v[4 * j] = x.x; v[4 * j + 1] = x.y; v[4 * j + 2] = x.z; v[4 * j + 3] = x.w;
                if (phi)  // the identity: row c, column 64 hc + 32 i + 4 j + e
#pragma unroll
                    for (int e = 0; e < 4; ++e) v[4 * j + e] = (c == 64 * hc + 32 * i + 4 * j + e) ? 1.f : 0.f;
            }
            store_half(i, v);
        }
        if (tb == 0) {
            for (int i = 0; i < 2 && i < nchunks; ++i) {
                issue_chunk(maps, stage_tiles(smem, i), sv, h, i, &sm.mbar_ld[i], GATES, phi);
                ++sm.ld_issued[i];
            }
        }

        // gam of the previous chunk for this thread's row, when that chunk's
        // state update still owes the Diag(gam) (a fast chunk)
        float gm_owed = 1.f;
        uint32_t ph_b = 0, ph_o = 0, ph_rdy = 0;
        for (int n = 0; n < nchunks; ++n) {
            const int s = n & 1;
            ChunkTiles st = stage_tiles(smem, s);
            bf16 *W16 = st.k;  // -W, in the k slot
            bf16 *T16 = reinterpret_cast<bf16 *>(st.w);
            bf16 *M16 = T16 + C * C;
            bf16 *U16 = st.v;  // after T (w . v)

            if (gated && tb == 0) {  // the chunk's output-gate rows into L2 while the chain runs
                tc::tma_prefetch_4d(&maps.g, 0, h, sv.map_t0 + n * C, sv.map_b);
                tc::tma_prefetch_4d(&maps.g, 64, h, sv.map_t0 + n * C, sv.map_b);
            }
            wait_stage(&sm.ready[s], ph_rdy, s);
            GB::sync();
            if (sm.abort) break;
            const bool slow = sm.slow[s] != 0;
            const float gm = sm.gamma[s][c];
            if (!slow) {
                // ---- WY solve of a fast chunk: A (k slot) and group A's diagonal-block
                // inverses (w slot) -> T16 (first half of the w tile), with the fp32
                // work area in the second half of the S16 area (the previous chunk's
                // O image may still be going out from the first half)
                wy_solve<NG, GB>(reinterpret_cast<const float *>(st.k), reinterpret_cast<float *>(G16), T16,
                                 reinterpret_cast<const float *>(st.w));
                tc::fence_async_smem();
            }
            // (the solve's work area and the state copy below take the S16
            // area: the previous chunk's O image has been read by now)
            if (tb == 0) tc::bulk_wait_read();
            GB::sync();

            // ---- the products that need no state (M = 64, N = 128, K = 64): T Gt
            // into O's columns (free until O = Qt S, issued once -W is read back)
            // and T (w . v) into U's; the decayed operands Qt, Gt, Kb (or Kt) go
            // out for the backward
            if (tb == 0) {
                if (a.ops) {
                    unsigned char *op = static_cast<unsigned char *>(a.ops) + (sv.cslot + n) * kOpsTileBytes;
                    tc::bulk_store(op, st.q, TILE);
                    tc::bulk_store(op + TILE, st.b, TILE);
                    tc::bulk_store(op + 2 * TILE, st.la, TILE);
                    tc::bulk_commit();
                }
                mma_tiles<true, false>(tmem + COL_O, T16, 64, st.b, 64, 4, ID64x128_K_MN, false);
                mma_tiles<true, false>(tmem + COL_U, T16, 64, st.v, 64, 4, ID64x128_K_MN, false);
                tc::commit(&sm.mbar_b);
            }
            // ---- meanwhile the chunk-start state: the owed Diag(gam) of the
            // previous chunk, and its bf16 copy
            for (int i = 0; i < 2; ++i) {
                float v[32];
                load_half(i, v);
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] *= gm_owed;
                store_half(i, v);  // (warp-collective: never behind a per-thread condition)
                put_half(i, v);
            }
            handoff();
            // ---- the state, T and M (and U, below) go out for the backward as
            // their shared-memory images
            if (tb == 0) {
                keep_state(n);
                if (a.intra) {
                    tc::bulk_store(keep_tile(n), T16, 2 * C * C * 2);
                    tc::bulk_commit();
                }
            }
            wait_on(&sm.mbar_b, ph_b);  // T Gt, T (w . v)
            {  // -W = -(T Gt) -> bf16 in the k slot
                Frag<8> f;
                ld_frag(tmem + lane_base + COL_O + 64 * hc, f);
                tc::wait_ld();
                store_frag_bf16<D, 8>(f, W16, 16 * p, 64 * hc, lane, -1.f);
            }
            handoff();
            // ---- U = T (w . v) + (-W) S first (the chain waits for it), then O = Qt S
            if (tb == 0) {
                mma_tiles<true, false>(tmem + COL_U, W16, 64, S16, D, 8, ID64x128_K_MN, true);
                tc::commit(&sm.mbar_b);
                if (with_o) mma_tiles<true, false>(tmem + COL_O, st.q, 64, S16, D, 8, ID64x128_K_MN, false);
                if (gated) tc::commit(&sm.mbar_o);
            }
            wait_on(&sm.mbar_b, ph_b);  // U
            {  // U -> bf16 in the v slot (w . v is consumed)
                Frag<8> f;
                ld_frag(tmem + lane_base + COL_U + 64 * hc, f);
                tc::wait_ld();
                store_frag_bf16<D, 8>(f, U16, 16 * p, 64 * hc, lane, 1.f);
            }
            if (gated) wait_on(&sm.mbar_o, ph_o);  // O = Qt S: the gate tile lands where S16 was
            handoff();
            if (sm.abort) break;
            if (tb == 0 && a.intra) {
                tc::bulk_store(keep_tile(n) + 2 * C * C * 2, U16, C * D * 2);
                tc::bulk_commit();
            }
            if (gated && tb == 0) {  // every product that reads S16 is complete
                tc::mbar_expect_tx(&sm.mbar_g, TILE);
                tc::tma_load_4d(G16, &maps.g, 0, h, sv.map_t0 + n * C, sv.map_b, &sm.mbar_g);
                tc::tma_load_4d(G16 + C * 64, &maps.g, 64, h, sv.map_t0 + n * C, sv.map_b, &sm.mbar_g);
                ++sm.g_issued;
            }
            // ---- slow chunk: S <- Diag(gam) S before adding Kt^T U
            if (slow) {
                for (int i = 0; i < 2; ++i) {
                    float v[32];
                    load_half(i, v);
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] *= gm;
                    store_half(i, v);
                }
                tc::fence_before();
                GB::sync();
                tc::fence_after();
            }
            // ---- O += M U (committed first: the O epilogue runs under the state
            // update) ; S += Kx^T U
            if (tb == 0) {
                if (with_o) mma_tiles<true, false>(tmem + COL_O, M16, 64, U16, 64, 4, ID64x128_K_MN, true);
                tc::commit(&sm.mbar_o);
                mma_tiles<false, false>(tmem + COL_S, st.la, 64, U16, 64, 4, IDESC_S, true);
                tc::commit(&sm.mbar_b);
            }
            wait_on(&sm.mbar_o, ph_o);
            gm_owed = slow ? 1.f : gm;  // a fast chunk's Diag(gam) is applied with the next bf16 copy
            if (a.states && with_o) {  // the state image (the S16 area) has gone out
                if (tb == 0) {
                    if (a.intra) tc::bulk_wait_read_but<1>();  // (all but the U tile's store)
                    else tc::bulk_wait_read();
                }
                GB::sync();
            }
            if (with_o) {  // O -> its bf16 image in the first half of the S16 area, stored by the TMA
                Frag<8> f;
                ld_frag(tmem + lane_base + COL_O + 64 * hc, f);
                tc::wait_ld();
                if (gated) {  // z = O / rms(O) * gamma * silu(g), row by row over both column halves
                    // (the RMS partials of the two column halves [2][64] in the q slot,
                    // whose last reader, O = Qt S, is complete; the fused epilogue
                    // keeps nothing for a backward pass)
                    float *rms_part = reinterpret_cast<float *>(st.q);
                    const int r0 = 16 * p + (lane >> 2);
                    float ss[2] = {0.f, 0.f};
#pragma unroll
                    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) ss[e >> 1] = fmaf(f[0][nt][e], f[0][nt][e], ss[e >> 1]);
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        ss[i] += __shfl_xor_sync(0xffffffffu, ss[i], 1);
                        ss[i] += __shfl_xor_sync(0xffffffffu, ss[i], 2);
                    }
                    if ((lane & 3) == 0) {
                        rms_part[hc * C + r0] = ss[0];
                        rms_part[hc * C + r0 + 8] = ss[1];
                    }
                    if (wait_on(&sm.mbar_g, ph_g) && tb == 0) ++sm.g_landed;
                    GB::sync();
                    float rs[2];
#pragma unroll
                    for (int i = 0; i < 2; ++i)
                        rs[i] = rsqrtf((rms_part[r0 + 8 * i] + rms_part[C + r0 + 8 * i]) * (1.f / D) + 1e-6f);
#pragma unroll
                    for (int nt = 0; nt < 8; ++nt) {
                        const int col = 64 * hc + 8 * nt + 2 * (lane & 3);
                        const float2 gmw = *reinterpret_cast<const float2 *>(a.gamma + col);
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const float2 gg = unpack_bf16(*reinterpret_cast<const uint32_t *>(G16 + swz<D>(r0 + 8 * i, col)));
                            f[0][nt][2 * i] *= rs[i] * gmw.x * gg.x / (1.f + __expf(-gg.x));
                            f[0][nt][2 * i + 1] *= rs[i] * gmw.y * gg.y / (1.f + __expf(-gg.y));
                        }
                    }
                }
                store_frag_bf16<D, 8>(f, O16, 16 * p, 64 * hc, lane, 1.f);
                tc::fence_async_smem();
            }
            wait_on(&sm.mbar_b, ph_b);  // S (and with it every read of the stage's tiles)
            tc::fence_before();
            GB::sync();
            // the last chunk of a packed sequence: its rows of o by the threads
            // (a box would reach into the next sequence's rows)
            const int Cn = min(C, sv.len - n * C);
            const bool o_rows = with_o && packed && Cn < C;
            if (o_rows) {
                bf16 *o = static_cast<bf16 *>(op);
                for (int id = tb; id < Cn * 16; id += NG) {
                    const int r = id >> 4, j = id & 15;
                    const uint4 val = *reinterpret_cast<const uint4 *>(O16 + (j >> 3) * (C * 64) + r * 64 +
                                                                       (((j & 7) ^ (r & 7)) << 3));
                    *reinterpret_cast<uint4 *>(o + ((sv.row0 + n * C + r) * a.H + h) * D + 8 * j) = val;
                }
                tc::fence_async_smem();
                GB::sync();
            }
            if (tb == 0) {
                if (with_o && !o_rows) {  // (tokens past the tensor's end are clipped)
                    tc::tma_store_4d(omap, O16, 0, h, sv.map_t0 + n * C, sv.map_b);
                    tc::tma_store_4d(omap, O16 + C * 64, 64, h, sv.map_t0 + n * C, sv.map_b);
                }
                tc::bulk_commit();  // (one group, possibly empty, so that the wait below skips exactly it)
                // the stage's T, M, U and operand images are out before the stage
                // is refilled; the O image may still be in flight (its area is
                // waited for before the next state copy)
                tc::bulk_wait_read_but<1>();
                if (n + 2 < nchunks) {  // (six whole-tile boxes: a short issue)
                    issue_chunk(maps, st, sv, h, n + 2, &sm.mbar_ld[s], GATES, phi);
                    ++sm.ld_issued[s];
                }
            }
        }
        if (tb == 0) tc::bulk_wait_read();  // (the last O image, in the S16 area)
        GB::sync();
        if (!sm.abort) {  // the final state: S_T and (when requested) its bf16 image
            tc::fence_after();
            for (int i = 0; i < 2; ++i) {
                float v[32];
                load_half(i, v);
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] *= gm_owed;
                if (STp) {
                    float4 *dst = reinterpret_cast<float4 *>(STp + (size_t)c * D + 64 * hc +
                                                             32 * i);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                }
                put_half(i, v);
            }
            if (a.states) {
                tc::fence_async_smem();
                GB::sync();
                if (tb == 0) keep_state(nchunks);
            }
        }
        if (tb == 0) tc::bulk_wait();
    }
    // Before the tensor memory is freed: each issuing thread's tensor-core work
    // has finished (a commit tracks all of it; immediate after a normal pass)
    // and, after an aborted pass, every tile load issued has landed (bounded).
    if (tid == 0 || tid == NG) {
        uint64_t *fin = &sm.mbar_fin[tid == 0 ? 0 : 1];
        tc::commit(fin);
        (void)tc::mbar_wait(fin, 0, wait_limit);
    }
    tc::fence_before();
    __syncthreads();
    if (tid == 0) {
        for (int i = 0; i < 2; ++i)
            for (; sm.ld_waited[i] < sm.ld_issued[i]; ++sm.ld_waited[i])
                (void)tc::mbar_wait(&sm.mbar_ld[i], (uint32_t)(sm.ld_waited[i] & 1), wait_limit);
        for (; sm.g_landed < sm.g_issued; ++sm.g_landed)
            (void)tc::mbar_wait(&sm.mbar_g, (uint32_t)(sm.g_landed & 1), wait_limit);
    }
    __syncthreads();
    if (warp == 0) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace cfwd_tc

cudaError_t launch_chunk_fwd_tc(const ChunkFwdArgs &a, cudaStream_t s) {
    cfwd_tc::FwdMaps m{};
    const int D = cfwd_tc::D;
    const int MB = a.cu_seqlens ? 1 : a.B;  // a packed batch is one [T, H, D] sequence of rows
    const bool vec_la = a.gates != kGatesGDN, vec_bw = a.gates == kGatesFull;  // (scalar gates: no maps)
    if (!token_tile_map(&m.q, a.q, MB, a.T, a.H, D) || !token_tile_map(&m.k, a.k, MB, a.T, a.H, D) ||
        (vec_la && !token_tile_map(&m.la, a.log_alpha, MB, a.T, a.H, D)) ||
        (vec_bw && !token_tile_map(&m.b, a.b, MB, a.T, a.H, D)) || !token_tile_map(&m.v, a.v, MB, a.T, a.H, D) ||
        (vec_bw && !token_tile_map(&m.w, a.w, MB, a.T, a.H, D)) ||
        (a.o && !token_tensor_map(&m.o, a.o, MB, a.T, a.H, D)) ||
        (a.out_gate && !token_tensor_map(&m.g, a.out_gate, MB, a.T, a.H, D)) ||
        (a.seg_P && !token_tensor_map(&m.qphi, a.seg_qphi, a.B, a.T, a.H, D)))
        return cudaErrorInvalidValue;
    if (a.seg_P && (a.seg_P < 2 || a.T % cfwd_tc::C || a.T / cfwd_tc::C < a.seg_P || a.cu_seqlens || a.states ||
                    a.gates != kGatesFull || !a.seg_loc || !a.seg_phi || !a.seg_qphi))
        return cudaErrorInvalidValue;
    if (a.out_gate && (a.states || !a.o || !a.gamma)) return cudaErrorInvalidValue;  // (inference path only)
    if (a.transition) return cudaErrorInvalidValue;  // (this kernel takes its transition passes by seg_P)
    using namespace cfwd_tc;
    auto kernel = a.seg_P                  ? chunk_fwd_tc_kernel<kGatesFull, kSegments>
                  : a.out_gate             ? chunk_fwd_tc_kernel<kGatesFull, kGated>
                  : a.gates == kGatesKDA   ? chunk_fwd_tc_kernel<kGatesKDA, kPlain>
                  : a.gates == kGatesGDN   ? chunk_fwd_tc_kernel<kGatesGDN, kPlain>
                                           : chunk_fwd_tc_kernel<kGatesFull, kPlain>;
    if (a.out_gate && a.gates != kGatesFull) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, BYTES);
    if (e != cudaSuccess) return e;
    const unsigned ctas = (unsigned)(a.B * a.H) * (a.seg_P ? 2u * a.seg_P - 1u : 1u);
    kernel<<<ctas, NT, BYTES, s>>>(a, m);
    return cudaGetLastError();
}

}  // namespace gdn2
