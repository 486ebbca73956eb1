// Reverse chunk pass of the backward for dk = dv = 128 with every chunk
// product on the fifth-generation tensor cores (tcgen05, accumulators in
// tensor memory).
//
// Same algebra as chunk_bwd.cu ("Why NVIDIA Gated DeltaNet-2 separates erase
// and write gates", section "Gated Delta Rule-2: per-channel erase/write
// split"; the gradients of the WY form follow from the laonpeople Gated
// DeltaNet page's chunk equations).  Tensor memory (512 columns x 128 lanes)
// holds, per CTA:
//   cols   0..127  R_A: dO U^T (0..63), nR U^T (64..127), then dQt
//   cols 128..255  R_B: -nR = T^T dU, then dGt
//   cols 256..383  R_C: dU, then dKb
//   cols 384..511  R_S: dSigma (128 key rows x 128 value columns, fp32)
// One thread issues four groups of MMAs per chunk; after each group the warps
// read the results back (16x256b shape for the 64-row products, which lands
// in the register layout of a warp-level m16n8 fragment; 32x32b rows for
// dSigma), form the next bf16 operands in shared memory, and hand over:
//   M1  dU = M^T dO + Kx D (committed first) ; dO U^T ; dSigma += Qt^T dO
//       (D = g . dSigma)
//   M2  T^T dU
//   M3  nR U^T ;  dGt = nR S^T ;  dKb = U D^T ;  dSigma += Gt^T nR
//   M4  dQt = dO S^T (+ dM Kb) ;  dGt += dA Kb ;  dKb += dA^T Gt + dM^T Qt
//       (dM as the sum of two bf16 tiles, its rounding and the remainder)
// (the Gram terms in M4 only on a fast chunk; a slow chunk takes them term by
// term in fp32, as in chunk_bwd.cu).  Work off the chain runs inside the
// products: dM and dv, dw during M3, the raw token rows and the dSigma.Sigma
// row sums during M4.  dQt, dGt and dKb then go to the fp32 staging tiles and
// the token-level gradients follow, four key channels per thread
// (chunk_bwd_common.cuh token_grads4).  Every wait on an mbarrier is bounded:
// on expiry the kernel records GDN2_ERR_TIMEOUT in the device status word,
// frees its tensor memory and returns.
#include "chunk_bwd_common.cuh"
#include "gdn2.h"
#include "tc_tiles.cuh"
#include "tma_host.h"

namespace gdn2 {
namespace cbwd_tc {

using namespace chunk;
using cbwd::BSmem;
using cbwd::BwdChunk;

constexpr int D = 128;
constexpr int NT = 512;  // 16 warps: four per tensor-memory sub-partition
using L = BSmem<D, D>;
using Chunk = BwdChunk<D, D, NT>;
constexpr int TILE_BYTES = C * D * 2;
constexpr int TM_BYTES = 2 * C * C * 2;

// TMA tensor maps of the token tensors read as tiles.
struct BwdMaps {
    CUtensorMap la, dO;
};
constexpr int BYTES = L::BYTES + 1024;  // + room to align the tiles to 1 KB

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t COL_A = 0, COL_B = 128, COL_C = 256, COL_S = 384;
// instruction descriptors: shape, then the majorness of A and B (MN = the
// operand is stored with its M (or N) index along the rows' contiguous axis)
constexpr uint32_t ID64x128_MN_MN = tc::idesc_bf16(64, 128, true, true);
constexpr uint32_t ID64x128_K_MN = tc::idesc_bf16(64, 128, false, true);
constexpr uint32_t ID64x128_K_K = tc::idesc_bf16(64, 128, false, false);
constexpr uint32_t ID64x64_K_K = tc::idesc_bf16(64, 64, false, false);
constexpr uint32_t ID128x128_MN_MN = tc::idesc_bf16(128, 128, true, true);

using tct::Frag;
using tct::dot8;
using tct::ld_frag;
using tct::mma_tiles;
using tct::store_frag_bf16;

// Decay of chunk n from its raw log_alpha tile (bf16, swizzled [64][D]):
// seg[s][c] = sum of log_alpha[., c] over the rows before row 4 s (lane =
// channel quad, warp = 4-row segment, as in the token-level gradients),
// gamma[c] = e^{L_end};
// true (and L in lam_ws, [64][D] fp32) when the chunk decays by more than
// e^{-kSpanGuard} in some channel.  Tokens past T read as zeros.
__device__ bool decay_sums(const bf16 *la, float (*seg)[D], float *gamma, int *slow_flag, float *lam_ws, int tid) {
    constexpr int P4 = Chunk::P4, R4 = Chunk::R4;
    const int c4 = 4 * (tid % Chunk::NQ), s4 = tid / Chunk::NQ;
    if (tid == 0) *slow_flag = 0;
    float2 s0 = make_float2(0.f, 0.f), s1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < R4; ++i) {
        const uint2 v = *reinterpret_cast<const uint2 *>(la + swz<D>(s4 * R4 + i, c4));
        s0 = __fadd2_rn(s0, unpack_bf16(v.x));
        s1 = __fadd2_rn(s1, unpack_bf16(v.y));
    }
    *reinterpret_cast<float4 *>(&seg[s4][c4]) = make_float4(s0.x, s0.y, s1.x, s1.y);
    __syncthreads();
    if (s4 == P4 - 1) {  // the last segment's warp: exclusive prefix sums in place, and L_end
        float4 t[P4];
#pragma unroll
        for (int s = 0; s < P4; ++s) t[s] = *reinterpret_cast<const float4 *>(&seg[s][c4]);
        float2 t0 = make_float2(0.f, 0.f), t1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int s = 0; s < P4; ++s) {
            *reinterpret_cast<float4 *>(&seg[s][c4]) = make_float4(t0.x, t0.y, t1.x, t1.y);
            t0 = __fadd2_rn(t0, make_float2(t[s].x, t[s].y));
            t1 = __fadd2_rn(t1, make_float2(t[s].z, t[s].w));
        }
        *reinterpret_cast<float4 *>(gamma + c4) = make_float4(__expf(t0.x), __expf(t0.y), __expf(t1.x), __expf(t1.y));
        if (fminf(fminf(t0.x, t0.y), fminf(t1.x, t1.y)) < -kSpanGuard) *slow_flag = 1;
    }
    __syncthreads();
    const bool slow = *slow_flag != 0;
    if (slow) {  // the exact path needs L at every token
        if (tid < D) {
            float lam = 0.f;
            for (int r = 0; r < C; ++r) {
                lam += __bfloat162float(la[swz<D>(r, tid)]);
                lam_ws[r * D + tid] = lam;
            }
        }
        __syncthreads();
    }
    return slow;
}

template <int GATES>
__global__ void __launch_bounds__(NT, 1) chunk_bwd_tc_kernel(ChunkBwdArgs a, const __grid_constant__ BwdMaps maps) {
    using Chunk = BwdChunk<D, D, NT, GATES>;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (tc::smem_addr(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(16) float s_seg[Chunk::P4][D];  // log_alpha sums over the 4-row segments of a chunk
    __shared__ __align__(16) float s_gamma[D];            // e^{L_end} of the chunk
    __shared__ int s_slow;
    __shared__ float s_dmd[C];
    __shared__ float s_dbw[C];  // scalar gates: per token, the sum of dw over the value channels
    __shared__ __align__(16) float s_rs[2][Chunk::NRS][D];  // by chunk parity: row sums of dSigma . Sigma (column quarters)
    __shared__ uint64_t mbar;
    __shared__ uint64_t mbar_ld[3];  // load groups A, B and the state image
    __shared__ uint64_t mbar_fin;    // the issuing thread's last tensor-core work, at the end
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;

    Chunk x(a, smem, nullptr, nullptr, s_dmd, s_rs[0]);
    x.dMlo16 = x.U16;  // dM's low-order part goes to the U slot after M3 (E3)
    x.s_dbw = s_dbw;
    const int tid = x.tid, warp = x.warp, lane = x.lane, bh = blockIdx.x;
    const ChunkTiles st = x.st;
    if (!x.sv.ok) {  // packed-sequence offsets out of range: nothing of this sequence is touched
        if (tid == 0) record_status(a.status, GDN2_ERR_INVALID_ARG);
        return;
    }
    const bool packed = a.cu_seqlens != nullptr;

    if (warp == 0) tc::tmem_alloc(&tmem_slot, kTmemCols);
    if (tid == 0) {
        tc::mbar_init(&mbar, 1);
        tc::mbar_init(&mbar_ld[0], 1);
        tc::mbar_init(&mbar_ld[1], 1);
        tc::mbar_init(&mbar_ld[2], 1);
        tc::mbar_init(&mbar_fin, 1);
        tc::fence_mbar_init();
        abort_flag = 0;
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = tmem_slot;

    // Thread <-> dSigma row c = 32 p + lane of sub-partition p; warps p,
    // p + 4, p + 8, p + 12 take the column quarters qc = 0..3.  For the 64-row
    // products the same warp reads rows 16 p .. 16 p + 15, columns 32 qc ...
    const int p = warp & 3, qc = warp >> 2, c = 32 * p + lane;
    const uint32_t lane_base = (uint32_t)(32 * p) << 16;
    const uint32_t t_srow = tmem + lane_base + COL_S + 32 * qc;
    // this thread's 32 columns of a swizzled [128][128] bf16 tile row c, as 4 x 8
    auto tile_row = [&](const bf16 *tile, int i) {
        return tile + (qc >> 1) * (D * 64) + c * 64 + (((4 * (qc & 1) + i) ^ (c & 7)) << 3);
    };

    {  // dSigma of the last chunk end = dS_T (or zero)
        float v[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 y = a.dS_T ? reinterpret_cast<const float4 *>(a.dS_T + (size_t)bh * D * D + (size_t)c * D +
                                                                       32 * qc)[i]
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
            v[4 * i] = y.x; v[4 * i + 1] = y.y; v[4 * i + 2] = y.z; v[4 * i + 3] = y.w;
        }
        tc::st_32x32b_x32(t_srow, v);
        tc::wait_st();
    }

    uint32_t phase = 0;
    const uint32_t wait_limit = a.wait_limit ? a.wait_limit : tc::kWaitLimit;
    // Wait for the MMAs committed last (all threads) ...
    auto mma_wait = [&]() {
        if (!tc::mbar_wait(&mbar, phase, wait_limit)) {
            abort_flag = 1;
            record_status(a.status, GDN2_ERR_TIMEOUT);
        }
        phase ^= 1;
        tc::fence_after();
    };
    // ... or commit the MMAs issued so far and wait for them.
    auto mma_done = [&]() {
        if (tid == 0) tc::commit(&mbar);
        mma_wait();
    };
    // Shared-memory operands written by the threads -> visible to the tensor
    // cores, and everybody's tensor-memory accesses ordered before the next MMA.
    auto handoff = [&]() {
        tc::fence_async_smem();
        tc::fence_before();
        __syncthreads();
        tc::fence_after();
    };

    // Tile loads, issued by one thread through the TMA and counted in bytes on
    // mbar_ld: group A = the forward's Qt, Gt, Kb (or Kt) and U, with the raw
    // log_alpha (into the k slot, for the decay sums) and dO as 64 x 64 boxes
    // of the tensor maps; group B = the forward's T, M; then the chunk-start
    // state on a barrier of its own (first needed by M3).  The forward stores
    // its tiles as images of shared memory, which come back as bulk copies.
    // They run one chunk ahead: group A of chunk n - 1 lands while chunk n's
    // token-level gradients are formed, group B and the state while chunk
    // n - 1's decay sums, E0 and first products run.
    uint32_t ph_ld[3] = {0, 0, 0};
    int ld_issued[3] = {0, 0, 0}, ld_landed[3] = {0, 0, 0};  // (thread 0: its loads, for the drain at the end)
    constexpr bool scalar_la = GATES == kGatesGDN;  // a scalar decay: its tile is filled after the loads
    auto issue_a = [&](int m) {
        tc::mbar_expect_tx(&mbar_ld[0], (scalar_la ? 5 : 6) * TILE_BYTES);
        const unsigned char *img = x.intra + (size_t)m * x.I_BYTES + TM_BYTES;
        const unsigned char *op = static_cast<const unsigned char *>(a.ops) + (x.sv.cslot + m) * kOpsTileBytes;
        const int t = x.sv.map_t0 + m * C, mb = x.sv.map_b;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int cx = 64 * half, off = half * C * 64;
            if (!scalar_la) tc::tma_load_4d(st.k + off, &maps.la, cx, x.h, t, mb, &mbar_ld[0]);
            tc::tma_load_4d(x.dO16 + off, &maps.dO, cx, x.h, t, mb, &mbar_ld[0]);
        }
        tc::bulk_load(st.q, op, TILE_BYTES, &mbar_ld[0]);
        tc::bulk_load(st.b, op + TILE_BYTES, TILE_BYTES, &mbar_ld[0]);
        tc::bulk_load(st.la, op + 2 * TILE_BYTES, TILE_BYTES, &mbar_ld[0]);
        tc::bulk_load(x.U16, img, TILE_BYTES, &mbar_ld[0]);
        ++ld_issued[0];
    };
    auto issue_b = [&](int m) {
        tc::mbar_expect_tx(&mbar_ld[1], TM_BYTES);
        tc::bulk_load(x.T16, x.intra + (size_t)m * x.I_BYTES, TM_BYTES, &mbar_ld[1]);
        tc::mbar_expect_tx(&mbar_ld[2], D * D * 2);
        tc::bulk_load(x.S16, x.states + (size_t)m * D * D, D * D * 2, &mbar_ld[2]);
        ++ld_issued[1];
        ++ld_issued[2];
    };
    auto wait_loads = [&](int g) {
        if (!tc::mbar_wait(&mbar_ld[g], ph_ld[g], wait_limit)) {
            abort_flag = 1;
            record_status(a.status, GDN2_ERR_TIMEOUT);
        } else {
            ++ld_landed[g];
        }
        ph_ld[g] ^= 1;
    };

    if (tid == 0 && x.nchunks > 0) {
        issue_a(x.nchunks - 1);
        issue_b(x.nchunks - 1);
    }
    for (int n = x.nchunks - 1; n >= 0; --n) {
        const int Cn = min(C, x.len - n * C);
        wait_loads(0);
        __syncthreads();
        if (abort_flag) break;
        if (scalar_la) {
            // the raw log_alpha tile from the scalar decay (zero past the sequence's end)
            const unsigned short *lsc = static_cast<const unsigned short *>(a.log_alpha);
            for (int id = tid; id < 2 * C * 8; id += NT) {
                const int blk = id / (C * 8), r = (id % (C * 8)) / 8, ch = id % 8;
                uint32_t v = r < Cn ? lsc[(x.row0 + (size_t)n * C + r) * a.H + x.h] : 0u;
                v |= v << 16;
                *reinterpret_cast<uint4 *>(st.k + blk * (C * 64) + r * 64 + ch * 8) = make_uint4(v, v, v, v);
            }
            __syncthreads();
        }
        if (packed && Cn < C) {
            // the last chunk of a packed sequence: the log_alpha and dO boxes reach
            // into the next sequence; its rows read as zero tokens
            for (int id = tid; id < 2 * 2 * (C - Cn) * 8; id += NT) {
                const int tl = id / (2 * (C - Cn) * 8), rem = id % (2 * (C - Cn) * 8);
                const int blk = rem / ((C - Cn) * 8), r = Cn + (rem % ((C - Cn) * 8)) / 8, ch = rem % 8;
                *reinterpret_cast<uint4 *>((tl ? x.dO16 : st.k) + blk * (C * 64) + r * 64 + ch * 8) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
            __syncthreads();
        }
        if (n > 0) x.prefetch_vw_l2(n - 1);
        // gam, the decay segment sums and (slow chunk) L from the raw log_alpha in the k slot
        const bool slow = decay_sums(st.k, s_seg, s_gamma, &s_slow, x.LAM, tid);

        // ---- E0: D = g . dSigma (g = gam on a fast chunk, else 1) as bf16 and
        // dSigma <- gam . dSigma; on the last chunk also the row sums of
        // dSigma . Sigma (Sigma = the final state) for dL_end
        {
            float v[32];
            tc::ld_32x32b_x32(t_srow, v);
            tc::wait_ld();
            const float gm = s_gamma[c], g = slow ? 1.f : gm;
            const float2 g2 = make_float2(g, g), gm2 = make_float2(gm, gm);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t u[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 t = __fmul2_rn(make_float2(v[8 * i + 2 * e], v[8 * i + 2 * e + 1]), g2);
                    u[e] = pack_bf16(t.x, t.y);
                }
                *reinterpret_cast<uint4 *>(const_cast<bf16 *>(tile_row(x.D16, i))) = make_uint4(u[0], u[1], u[2], u[3]);
            }
            if (n == x.nchunks - 1) {
                const bf16 *sig = x.states + (size_t)(n + 1) * D * D;
                float rs = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) rs += dot8(v + 8 * i, *reinterpret_cast<const uint4 *>(tile_row(sig, i)));
                s_rs[n & 1][qc][c] = rs;
            }
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                const float2 t = __fmul2_rn(make_float2(v[i], v[i + 1]), gm2);
                v[i] = t.x;
                v[i + 1] = t.y;
            }
            tc::st_32x32b_x32(t_srow, v);
            tc::wait_st();
        }
        wait_loads(1);  // group B: T, M
        handoff();
        if (abort_flag) break;

        // ---- M1: dU = M^T dO + Kx D ; dO U^T ; dSigma += Qt^T dO
        // (dU is committed first: dO U^T and Qt^T dO run under E1, and M2's
        // commit covers them)
        if (tid == 0) {
            mma_tiles<false, false>(tmem + COL_C, x.M16, 64, x.dO16, 64, 4, ID64x128_MN_MN, false);
            mma_tiles<true, false>(tmem + COL_C, st.la, 64, x.D16, D, 8, ID64x128_K_MN, true);
            tc::commit(&mbar);
            mma_tiles<true, true>(tmem + COL_A, x.dO16, 64, x.U16, 64, 8, ID64x64_K_K, false);
            mma_tiles<false, false>(tmem + COL_S, st.q, 64, x.dO16, 64, 4, ID128x128_MN_MN, true);
        }
        mma_wait();
        // ---- E1: dU -> bf16 (all warps, column quarters)
        {
            Frag<4> f;
            ld_frag(tmem + lane_base + COL_C + 32 * qc, f);
            tc::wait_ld();
            store_frag_bf16<D, 4>(f, x.dU16, 16 * p, 32 * qc, lane, 1.f);
        }
        handoff();
        if (abort_flag) break;

        // ---- M2: T^T dU
        if (tid == 0) mma_tiles<false, false>(tmem + COL_B, x.T16, 64, x.dU16, 64, 4, ID64x128_MN_MN, false);
        mma_done();
        // ---- E2: nR = -T^T dU -> bf16
        {
            Frag<4> f;
            ld_frag(tmem + lane_base + COL_B + 32 * qc, f);
            tc::wait_ld();
            store_frag_bf16<D, 4>(f, x.nR16, 16 * p, 32 * qc, lane, -1.f);
        }
        wait_loads(2);  // the chunk-start state S
        handoff();
        if (abort_flag) break;

        // ---- M3: nR U^T ; dGt = nR S^T ; dKb = U D^T ; dSigma += Gt^T nR
        if (tid == 0) {
            mma_tiles<true, true>(tmem + COL_A + 64, x.nR16, 64, x.U16, 64, 8, ID64x64_K_K, false);
            mma_tiles<true, true>(tmem + COL_B, x.nR16, 64, x.S16, D, 8, ID64x128_K_K, false);
            mma_tiles<true, true>(tmem + COL_C, x.U16, 64, x.D16, D, 8, ID64x128_K_K, false);
            mma_tiles<false, false>(tmem + COL_S, st.b, 64, x.nR16, 64, 4, ID128x128_MN_MN, true);
            tc::commit(&mbar);
        }
        // While the tensor cores run: dM = strict_lower(dO U^T) from M1's columns,
        // with its diagonal kept aside in fp32 (warps 8..15; M3 writes other
        // columns) -- the diagonal of M carries no decay factor, so its gradient
        // goes straight to dq and dk and stays out of the Gram products -- and
        // dv, dw from nR and the global v, w (warps 1..15).
        if (qc >= 2) {
            Frag<4> f;
            ld_frag(tmem + lane_base + COL_A + 32 * (qc - 2), f);
            tc::wait_ld();
            const int r0 = 16 * p + (lane >> 2);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = r0 + (e >> 1) * 8, i = 32 * (qc - 2) + 8 * nt + 2 * (lane & 3) + (e & 1);
                    if (i == r) s_dmd[r] = f[0][nt][e];
                    if (i >= r) f[0][nt][e] = 0.f;
                }
            store_frag_bf16<64, 4>(f, x.dM16, 16 * p, 32 * (qc - 2), lane, 1.f);
        }
        x.template dvdw<32>(n, Cn);
        mma_wait();
        // ---- E3: dA = strict_lower(nR U^T) -> bf16 (warps with qc < 2); the
        // low-order part dM - bf16(dM) of dM (still in M1's columns) -> bf16 in
        // the U slot, which M3 was the last to read (warps with qc >= 2).  dM's
        // entries reach tens, and its bf16 rounding alone would move the
        // largest dq and dk entries by a few hundredths; with the second term
        // dM Kb and dM^T Qt carry about 16 significant bits.
        {
            Frag<4> f;
            const int j = 32 * (qc & 1);
            ld_frag(tmem + lane_base + COL_A + (qc < 2 ? 64 : 0) + j, f);
            tc::wait_ld();
            const int r0 = 16 * p + (lane >> 2);
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = r0 + (e >> 1) * 8, i = j + 8 * nt + 2 * (lane & 3) + (e & 1);
                    const float y = f[0][nt][e];
                    f[0][nt][e] = i >= r ? 0.f : (qc < 2 ? y : y - __bfloat162float(__float2bfloat16_rn(y)));
                }
            store_frag_bf16<64, 4>(f, qc < 2 ? x.dA16 : x.U16, 16 * p, j, lane, 1.f);
        }
        handoff();
        if (abort_flag) break;

        // ---- M4: dQt = dO S^T (+ dM Kb) ; dGt += dA Kb ; dKb += dA^T Gt + dM^T Qt
        if (tid == 0) {
            mma_tiles<true, true>(tmem + COL_A, x.dO16, 64, x.S16, D, 8, ID64x128_K_K, false);
            if (!slow) {
                mma_tiles<true, false>(tmem + COL_A, x.dM16, 64, st.la, 64, 4, ID64x128_K_MN, true);
                mma_tiles<true, false>(tmem + COL_A, x.U16, 64, st.la, 64, 4, ID64x128_K_MN, true);  // dM lo
                mma_tiles<true, false>(tmem + COL_B, x.dA16, 64, st.la, 64, 4, ID64x128_K_MN, true);
                mma_tiles<false, false>(tmem + COL_C, x.dA16, 64, st.b, 64, 4, ID64x128_MN_MN, true);
                mma_tiles<false, false>(tmem + COL_C, x.dM16, 64, st.q, 64, 4, ID64x128_MN_MN, true);
                mma_tiles<false, false>(tmem + COL_C, x.U16, 64, st.q, 64, 4, ID64x128_MN_MN, true);  // dM lo
            }
            tc::commit(&mbar);
        }
        typename Chunk::RawRows4 raw;
        x.load_rows4(raw, n, Cn);  // while the tensor cores run
        // ---- row sums of dSigma . Sigma for chunk n - 1 (dSigma is now its
        // chunk-end gradient, Sigma = this chunk's start state S), also inside M4
        if (n > 0) {
            float v[32];
            tc::ld_32x32b_x32(t_srow, v);
            tc::wait_ld();
            float rs = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) rs += dot8(v + 8 * i, *reinterpret_cast<const uint4 *>(tile_row(x.S16, i)));
            s_rs[(n - 1) & 1][qc][c] = rs;
        }
        __syncthreads();  // every read of S16 is done before E4 stages dQt over it
        mma_wait();
        // ---- E4: dQt, dGt, dKb -> fp32 staging (the S, D and T/M/dU regions are dead)
        {
            Frag<4> f;
            ld_frag(tmem + lane_base + COL_A + 32 * qc, f);
            tc::wait_ld();
            cbwd::store_stage<D, 4>(f, x.DQT, 16 * p, 32 * qc, lane);
            ld_frag(tmem + lane_base + COL_B + 32 * qc, f);
            tc::wait_ld();
            cbwd::store_stage<D, 4>(f, x.DGT, 16 * p, 32 * qc, lane);
            ld_frag(tmem + lane_base + COL_C + 32 * qc, f);
            tc::wait_ld();
            cbwd::store_stage<D, 4>(f, x.DKB, 16 * p, 32 * qc, lane);
        }
        // (every generic access of a tile is fenced against the TMA before it is refilled)
        tc::fence_async_smem();
        tc::fence_before();
        __syncthreads();
        if (abort_flag) break;

        if (slow) {
            x.slow_grams(n, Cn);
            tc::fence_async_smem();
            __syncthreads();
        }
        if (n > 0 && tid == 0) issue_a(n - 1);  // the token, dO and U slots are free now
        x.s_rs = s_rs[n & 1];
        // (the v slot's nR is consumed: its first 8 KB take the segment sums of
        // dL).  Group B and the state of chunk n - 1 load once the staging tiles
        // in the S and T/M regions are read, during the reverse cumulative sum.
        x.token_grads4(n, Cn, slow, raw, s_seg, reinterpret_cast<float (*)[D]>(st.v), [&] {
            if (n > 0 && tid == 0) issue_b(n - 1);
        });
    }

    if (a.dS0 && !abort_flag) {
        tc::fence_after();
        float v[32];
        tc::ld_32x32b_x32(t_srow, v);
        tc::wait_ld();
        float4 *dst = reinterpret_cast<float4 *>(a.dS0 + (size_t)bh * D * D + (size_t)c * D + 32 * qc);
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
    // Before the tensor memory is freed: the issuing thread's tensor-core work
    // has finished (a commit tracks all of it; immediate after a normal pass)
    // and, after an aborted pass, every tile load issued has landed (bounded).
    if (tid == 0) {
        tc::commit(&mbar_fin);
        (void)tc::mbar_wait(&mbar_fin, 0, wait_limit);
        for (int g = 0; g < 3; ++g)
            for (; ld_landed[g] < ld_issued[g]; ++ld_landed[g])
                (void)tc::mbar_wait(&mbar_ld[g], (uint32_t)(ld_landed[g] & 1), wait_limit);
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace cbwd_tc

cudaError_t launch_chunk_bwd_tc(const ChunkBwdArgs &a, cudaStream_t s) {
    cbwd_tc::BwdMaps m;
    const int MB = a.cu_seqlens ? 1 : a.B;  // a packed batch is one [T, H, D] sequence of rows
    if ((a.gates != kGatesGDN && !token_tensor_map(&m.la, a.log_alpha, MB, a.T, a.H, cbwd_tc::D)) ||
        !token_tensor_map(&m.dO, a.dO, MB, a.T, a.H, cbwd_tc::D))
        return cudaErrorInvalidValue;
    auto kernel = a.gates == kGatesKDA   ? cbwd_tc::chunk_bwd_tc_kernel<kGatesKDA>
                  : a.gates == kGatesGDN ? cbwd_tc::chunk_bwd_tc_kernel<kGatesGDN>
                                         : cbwd_tc::chunk_bwd_tc_kernel<kGatesFull>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, cbwd_tc::BYTES);
    if (e != cudaSuccess) return e;
    kernel<<<(unsigned)(a.B * a.H), cbwd_tc::NT, cbwd_tc::BYTES, s>>>(a, m);
    return cudaGetLastError();
}

}  // namespace gdn2
