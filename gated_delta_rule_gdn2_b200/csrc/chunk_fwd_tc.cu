// Chunk-parallel forward for dk = dv = 128 with every chunk product on the
// fifth-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// Same algebra as chunk_fwd.cu ("Why NVIDIA Gated DeltaNet-2 separates erase
// and write gates", section "Gated Delta Rule-2: per-channel erase/write
// split"; WY form from the laonpeople Gated DeltaNet page): per chunk
//   A = Gt Kb^T, M = Qt Kb^T,  T = (I + A)^{-1},
//   U = T (w . v) - (T Gt) S,   O = Qt S + M U,   S <- Diag(gam) (S + Kb^T U).
// The fp32 state S lives in TMEM (128 lanes = key channels x 128 columns)
// for the whole sequence.  Per chunk one thread issues four MMA groups:
//   the two Grams (M = N = 64, K = 128);
//   T (w . v) into U's columns and T Gt (M = 64, N = 128, K = 64);
//   U += (-W) S and O = Qt S (K = 128, bf16 S copy in shared memory as B);
//   S += Kb^T U (M = 128) and O += M U,
// and between them the warps read the results back with the 16x256b TMEM
// load shape (the register layout of a warp-level m16n8 fragment) to form
// the next bf16 operands: A in fp32 for the WY solve (TF32 tensor-core levels
// on fp32 16x16 diagonal blocks, chunk_common.cuh), M, -W and U in bf16.  S is
// scaled by gam in TMEM (32x32b load/store) and copied to bf16 for the next
// chunk.  A chunk whose decay spans more than e^{-64} takes its Grams term by
// term in fp32 inside the shared intra-chunk stage.  Tiles arrive by TMA and
// the tiles kept for the backward leave as bulk stores.  Every wait on an
// mbarrier is bounded: on expiry the kernel records GDN2_ERR_TIMEOUT in the
// device status word, frees its tensor memory and returns.
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

struct Small {
    IntraShared<D> intra;
    uint64_t mbar[1];     // MMA completion
    uint64_t mbar_ld[2];  // tile loads of stage 0 and 1
    uint32_t tmem;
    int abort;
};
constexpr int BYTES = OSMALL + (int)sizeof(Small);
static_assert(BYTES <= 232448, "shared memory per block");

// Tensor memory: U (Uv, then + (-W) S), O (Qt S, then + M U), the state S
// (fp32, 128 key rows x 128 value columns) and a work region for the Grams
// (A | M, 64 columns each) and then T Gt.
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

// TMA tensor maps of the six token tensors.
struct FwdMaps {
    CUtensorMap q, k, la, b, v, w;
};

// Chunk n's six token tiles into a stage (one thread; 64 x 64 boxes, two per
// tile), completion counted in bytes on the stage's mbarrier.
__device__ __forceinline__ void issue_chunk(const FwdMaps &m, ChunkTiles st, int b, int h, int n, uint64_t *mbar) {
    tc::mbar_expect_tx(mbar, 6 * TILE);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int cx = 64 * half, off = half * C * 64;
        tc::tma_load_4d(st.q + off, &m.q, cx, h, n * C, b, mbar);
        tc::tma_load_4d(st.k + off, &m.k, cx, h, n * C, b, mbar);
        tc::tma_load_4d(st.la + off, &m.la, cx, h, n * C, b, mbar);
        tc::tma_load_4d(st.b + off, &m.b, cx, h, n * C, b, mbar);
        tc::tma_load_4d(st.v + off, &m.v, cx, h, n * C, b, mbar);
        tc::tma_load_4d(st.w + off, &m.w, cx, h, n * C, b, mbar);
    }
}

__global__ void __launch_bounds__(NTHR, 1) chunk_fwd_tc_kernel(ChunkFwdArgs a, const __grid_constant__ FwdMaps maps) {
    extern __shared__ __align__(1024) unsigned char smem[];
    Small &sm = *reinterpret_cast<Small *>(smem + OSMALL);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tc::smem_addr(smem) & 1023u) {  // the operand atoms need 1 KB alignment
        if (tid == 0) record_status(a.status, GDN2_ERR_CUDA);
        return;
    }
    const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
    const int nchunks = (a.T + C - 1) / C;
    const bool with_o = a.o != nullptr;
    auto keep_tile = [&](int n) {
        return static_cast<unsigned char *>(a.intra) + ((size_t)bh * nchunks + n) * intra_tile_bytes(D);
    };
    float *lam_ws = a.ws ? a.ws + (size_t)bh * a.ws_stride : nullptr;
    bf16 *S16 = reinterpret_cast<bf16 *>(smem + OS16);

    if (warp == 0) tc::tmem_alloc(&sm.tmem, kTmemCols);
    if (tid == 0) {
        tc::mbar_init(&sm.mbar[0], 1);
        tc::mbar_init(&sm.mbar_ld[0], 1);
        tc::mbar_init(&sm.mbar_ld[1], 1);
        tc::fence_mbar_init();
        sm.abort = 0;
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = sm.tmem;

    // Thread <-> state row c = 32 p + lane of sub-partition p; warps p and
    // p + 4 share the rows and take column halves hc = 0, 1.
    const int p = warp & 3, hc = warp >> 2, c = 32 * p + lane;
    const uint32_t t_row = tmem + ((uint32_t)(32 * p) << 16) + COL_S + 64 * hc;

    // bf16 copy of this thread's 64 state values into S16
    auto put_state = [&](const float (&v)[64]) {
        bf16 *row = S16 + hc * (D * 64) + c * 64;
#pragma unroll
        for (int q8 = 0; q8 < 8; ++q8) {
            uint4 u;
            u.x = pack_bf16(v[8 * q8 + 0], v[8 * q8 + 1]);
            u.y = pack_bf16(v[8 * q8 + 2], v[8 * q8 + 3]);
            u.z = pack_bf16(v[8 * q8 + 4], v[8 * q8 + 5]);
            u.w = pack_bf16(v[8 * q8 + 6], v[8 * q8 + 7]);
            *reinterpret_cast<uint4 *>(row + ((q8 ^ (c & 7)) << 3)) = u;
        }
    };
    // The chunk-boundary state n (when requested) as the image of S16, by one
    // thread after the writers' proxy fence and a barrier.
    auto keep_state = [&](int n) {
        if (a.states) {
            tc::bulk_store(static_cast<bf16 *>(a.states) + ((size_t)bh * (nchunks + 1) + n) * D * D, S16, D * D * 2);
            tc::bulk_commit();
        }
    };
    auto load_state = [&](float (&v)[64]) {
        tc::ld_32x32b_x32(t_row, *reinterpret_cast<float(*)[32]>(&v[0]));
        tc::ld_32x32b_x32(t_row + 32, *reinterpret_cast<float(*)[32]>(&v[32]));
        tc::wait_ld();
    };
    auto store_state = [&](const float (&v)[64]) {
        tc::st_32x32b_x32(t_row, *reinterpret_cast<const float(*)[32]>(&v[0]));
        tc::st_32x32b_x32(t_row + 32, *reinterpret_cast<const float(*)[32]>(&v[32]));
        tc::wait_st();
    };

    // ---- initial state into TMEM and S16
    {
        float v[64];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float4 x = a.S0 ? reinterpret_cast<const float4 *>(a.S0 + (size_t)bh * D * D + (size_t)c * D +
                                                                     64 * hc)[i]
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
            v[4 * i] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z; v[4 * i + 3] = x.w;
        }
        store_state(v);
        put_state(v);
    }
    tc::fence_async_smem();
    tc::fence_before();
    __syncthreads();
    if (tid == 0) {
        keep_state(0);
        issue_chunk(maps, stage_tiles(smem, 0), b, h, 0, &sm.mbar_ld[0]);
        if (nchunks > 1) issue_chunk(maps, stage_tiles(smem, 1), b, h, 1, &sm.mbar_ld[1]);
    }

    uint32_t ph_mma = 0, ph_ld[2] = {0, 0};
    // Commit the MMAs issued so far (thread 0) and wait for them (all threads).
    auto mma_done = [&]() {
        if (tid == 0) tc::commit(&sm.mbar[0]);
        if (!tc::mbar_wait(&sm.mbar[0], ph_mma)) {
            sm.abort = 1;
            record_status(a.status, GDN2_ERR_TIMEOUT);
        }
        ph_mma ^= 1;
        tc::fence_after();
    };
    // Shared-memory operands written by the threads -> visible to the tensor cores.
    auto handoff = [&]() {
        tc::fence_async_smem();
        tc::fence_before();
        __syncthreads();
        tc::fence_after();
    };
    const uint32_t lane_base = (uint32_t)(32 * p) << 16;  // this warp's 16 rows of a 64-row product

    for (int n = 0; n < nchunks; ++n) {
        ChunkTiles st = stage_tiles(smem, n & 1);
        float *A32 = reinterpret_cast<float *>(st.k);  // k and w slots are free after the prep
        float *T32 = reinterpret_cast<float *>(st.w);
        bf16 *W16 = reinterpret_cast<bf16 *>(A32);     // -W, after the solve
        bf16 *T16 = reinterpret_cast<bf16 *>(T32);
        bf16 *M16 = T16 + C * C;
        bf16 *U16 = st.v;                              // after Uv

        if (!tc::mbar_wait(&sm.mbar_ld[n & 1], ph_ld[n & 1])) {
            sm.abort = 1;
            record_status(a.status, GDN2_ERR_TIMEOUT);
        }
        ph_ld[n & 1] ^= 1;
        __syncthreads();
        if (sm.abort) break;
        // decay prep and w . v; a slow chunk also takes its Grams term by term and
        // its WY solve here, a fast chunk continues below
        const bool slow = intra_chunk<D, D>(st, A32, T32, sm.intra, lam_ws, false, false, /*grams_ext=*/true);
        if (!slow) {
            // ---- Grams on the tensor cores: A = Gt Kb^T, M = Qt Kb^T (M = N = 64, K = 128)
            handoff();
            if (tid == 0) {
                mma_tiles<true, true>(tmem + COL_G, st.b, 64, st.la, 64, 8, ID64x64_K_K, false);
                mma_tiles<true, true>(tmem + COL_G + 64, st.q, 64, st.la, 64, 8, ID64x64_K_K, false);
            }
            mma_done();
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
                        *reinterpret_cast<float2 *>(A32 + r * C + i) =
                            make_float2(i < r ? f[0][nt][2 * h2] : 0.f, i + 1 < r ? f[0][nt][2 * h2 + 1] : 0.f);
                    }
            }
            __syncthreads();
            wy_solve<NTHR>(A32, T32);
            {  // M (lower with the diagonal) -> bf16, past T16
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
        handoff();
        if (sm.abort) break;

        // ---- Uv = T (w . v) and T Gt on the tensor cores (M = 64, N = 128, K = 64)
        if (tid == 0) {
            mma_tiles<true, false>(tmem + COL_U, T16, 64, st.v, 64, 4, ID64x128_K_MN, false);
            mma_tiles<true, false>(tmem + COL_G, T16, 64, st.b, 64, 4, ID64x128_K_MN, false);
        }
        mma_done();
        {  // -W = -(T Gt) -> bf16 in the k slot
            Frag<8> f;
            ld_frag(tmem + lane_base + COL_G + 64 * hc, f);
            tc::wait_ld();
            store_frag_bf16<D, 8>(f, W16, 16 * p, 64 * hc, lane, -1.f);
        }
        handoff();

        // ---- U = Uv + (-W) S and O = Qt S on the tensor cores; T and M (and U,
        // below) go out for the backward as their shared-memory images
        if (tid == 0) {
            if (a.intra) {
                tc::bulk_store(keep_tile(n), T16, 2 * C * C * 2);
                tc::bulk_commit();
            }
            mma_tiles<true, false>(tmem + COL_U, W16, 64, S16, D, 8, ID64x128_K_MN, true);
            if (with_o) mma_tiles<true, false>(tmem + COL_O, st.q, 64, S16, D, 8, ID64x128_K_MN, false);
        }
        mma_done();
        {  // U -> bf16 in the v slot (w . v is consumed)
            Frag<8> f;
            ld_frag(tmem + lane_base + COL_U + 64 * hc, f);
            tc::wait_ld();
            store_frag_bf16<D, 8>(f, U16, 16 * p, 64 * hc, lane, 1.f);
        }
        if (tid == 0) tc::bulk_wait_read();  // the previous state image is out: S16 may be rewritten below
        handoff();
        if (sm.abort) break;

        if (tid == 0 && a.intra) {
            tc::bulk_store(keep_tile(n) + 2 * C * C * 2, U16, C * D * 2);
            tc::bulk_commit();
        }
        // ---- slow chunk: S <- Diag(gam) S before adding Kt^T U
        if (slow) {
            float v[64];
            load_state(v);
            const float gm = sm.intra.gamma[c];
#pragma unroll
            for (int i = 0; i < 64; ++i) v[i] *= gm;
            store_state(v);
            tc::fence_before();
            __syncthreads();
            tc::fence_after();
        }
        // ---- S += Kx^T U ; O += M U
        if (tid == 0) {
            mma_tiles<false, false>(tmem + COL_S, st.la, 64, U16, 64, 4, IDESC_S, true);
            if (with_o) mma_tiles<true, false>(tmem + COL_O, M16, 64, U16, 64, 4, ID64x128_K_MN, true);
        }
        mma_done();
        if (with_o) {  // O -> o (bf16), straight from the fragment layout
            Frag<8> f;
            ld_frag(tmem + lane_base + COL_O + 64 * hc, f);
            tc::wait_ld();
            const int rl = 16 * p + (lane >> 2);
            bf16 *o = static_cast<bf16 *>(a.o);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int t = n * C + rl + 8 * half;
                if (t < a.T) {
                    bf16 *orow = o + (((size_t)b * a.T + t) * a.H + h) * D + 64 * hc;
#pragma unroll
                    for (int nt = 0; nt < 8; ++nt)
                        *reinterpret_cast<uint32_t *>(orow + 8 * nt + 2 * (lane & 3)) =
                            pack_bf16(f[0][nt][2 * half], f[0][nt][2 * half + 1]);
                }
            }
        }

        // ---- S <- Diag(gam) S (fast chunk), bf16 copy for the next chunk
        {
            float v[64];
            load_state(v);
            if (!slow) {
                const float gm = sm.intra.gamma[c];
#pragma unroll
                for (int i = 0; i < 64; ++i) v[i] *= gm;
                store_state(v);
            }
            put_state(v);
        }
        tc::fence_async_smem();
        tc::fence_before();
        __syncthreads();
        if (tid == 0) {
            // this stage's T, M and U images are out before the stage is refilled
            tc::bulk_wait_read();
            if (n + 2 < nchunks) issue_chunk(maps, st, b, h, n + 2, &sm.mbar_ld[n & 1]);
            keep_state(n + 1);
        }
    }
    if (tid == 0) tc::bulk_wait();
    __syncthreads();

    if (a.S_T && !sm.abort) {
        tc::fence_after();
        float v[64];
        load_state(v);
        float4 *dst = reinterpret_cast<float4 *>(a.S_T + (size_t)bh * D * D + (size_t)c * D + 64 * hc);
#pragma unroll
        for (int i = 0; i < 16; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 0) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace cfwd_tc

cudaError_t launch_chunk_fwd_tc(const ChunkFwdArgs &a, cudaStream_t s) {
    cfwd_tc::FwdMaps m;
    const int D = cfwd_tc::D;
    if (!token_tensor_map(&m.q, a.q, a.B, a.T, a.H, D) || !token_tensor_map(&m.k, a.k, a.B, a.T, a.H, D) ||
        !token_tensor_map(&m.la, a.log_alpha, a.B, a.T, a.H, D) || !token_tensor_map(&m.b, a.b, a.B, a.T, a.H, D) ||
        !token_tensor_map(&m.v, a.v, a.B, a.T, a.H, D) || !token_tensor_map(&m.w, a.w, a.B, a.T, a.H, D))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(cfwd_tc::chunk_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         cfwd_tc::BYTES);
    if (e != cudaSuccess) return e;
    cfwd_tc::chunk_fwd_tc_kernel<<<(unsigned)(a.B * a.H), chunk::NTHR, cfwd_tc::BYTES, s>>>(a, m);
    return cudaGetLastError();
}

}  // namespace gdn2
