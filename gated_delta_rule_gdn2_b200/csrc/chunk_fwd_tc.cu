// Chunk-parallel forward for dk = dv = 128 with the inter-chunk state
// propagation on the fifth-generation tensor cores (tcgen05, accumulators in
// tensor memory).
//
// Same algebra as chunk_fwd.cu ("Why NVIDIA Gated DeltaNet-2 separates erase
// and write gates", section "Gated Delta Rule-2: per-channel erase/write
// split"; WY form from the laonpeople Gated DeltaNet page): per chunk
//   U = Uv - W S,   O = Qt S + M U,   S <- Diag(gam) (S + Kb^T U).
// The fp32 state S lives in TMEM (128 lanes = key channels x 128 columns)
// for the whole sequence.  Per chunk one thread issues
//   D_W = (-W) S   and   D_Q = Qt S     (two M=64, N=128, K=128 MMAs, bf16 S
//                                        copy in shared memory as operand B)
//   S  += Kb^T U                        (M=128, N=128, K=64, accumulating in TMEM)
// and the warps read D_W / D_Q back with the 16x256b TMEM load shape, which
// lands in the register layout of the warp-level m16n8 products that form Uv
// and M U.  S is scaled by gam in TMEM (32x32b load/store) and copied to bf16
// for the next chunk.  The intra-chunk stage (decay prefix, operands, Grams,
// WY solve, W and Uv) is shared with the other kernels (chunk_common.cuh).
// Every wait on the MMA completion barrier is bounded: on expiry the kernel
// records GDN2_ERR_TIMEOUT in the device status word, frees its tensor memory
// and returns.
#include "chunk_common.cuh"
#include "gdn2.h"
#include "launch.h"
#include "tc.cuh"
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
    uint64_t mbar[2];
    uint64_t mbar_ld[2];  // tile loads of stage 0 and 1
    uint32_t tmem;
    int abort;
};
constexpr int BYTES = OSMALL + (int)sizeof(Small);
static_assert(BYTES <= 232448, "shared memory per block");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t COL_W = 0, COL_Q = 128, COL_S = 256;
constexpr uint32_t IDESC_WQ = tc::idesc_bf16(64, 128, false, true);  // A K-major, B MN-major
constexpr uint32_t IDESC_S = tc::idesc_bf16(128, 128, true, true);   // A, B MN-major

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
        tc::mbar_init(&sm.mbar[1], 1);
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

    uint32_t ph0 = 0, ph1 = 0, ph_ld[2] = {0, 0};
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
        const bool slow = intra_chunk<D, D>(st, A32, T32, sm.intra, lam_ws, false);

        // ---- Uv = T WV (warps 0..3, registers) ; -W = -T Gt (warps 4..7, shared)
        float acc[1][16][4];
        zero(acc);
        if (warp < 4) {
            warp_gemm<1, 16, true, false, 64, D>(acc, T16, 16 * warp, st.v, 0, C, lane);
        } else {
            warp_gemm<1, 16, true, false, 64, D>(acc, T16, 16 * p, st.b, 0, C, lane);
            store_tile_bf16<16, D>(acc, W16, 16 * p, lane, -1.f);
        }
        tc::fence_async_smem();
        __syncthreads();

        // ---- D_W = -W S, D_Q = Qt S on the tensor cores; T and M (and U,
        // below) go out for the backward as their shared-memory images
        if (tid == 0) {
            if (a.intra) {
                tc::bulk_store(keep_tile(n), T16, 2 * C * C * 2);
                tc::bulk_commit();
            }
            tc::fence_after();
            const uint32_t sS = tc::smem_addr(S16), sW = tc::smem_addr(W16), sQ = tc::smem_addr(st.q);
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const uint32_t koff = (s >> 2) * 8192 + (s & 3) * 32;
                const uint64_t bd = tc::sdesc(sS + s * 2048, D * 128, 1024);
                tc::mma_bf16(tmem + COL_W, tc::sdesc(sW + koff, 16, 1024), bd, IDESC_WQ, s > 0);
                if (with_o) tc::mma_bf16(tmem + COL_Q, tc::sdesc(sQ + koff, 16, 1024), bd, IDESC_WQ, s > 0);
            }
            tc::commit(&sm.mbar[0]);
        }
        if (!tc::mbar_wait(&sm.mbar[0], ph0)) {
            sm.abort = 1;
            record_status(a.status, GDN2_ERR_TIMEOUT);
        }
        ph0 ^= 1;
        tc::fence_after();

        // ---- U = Uv + D_W (warps 0..3) -> bf16 ; O starts as D_Q (warps 4..7)
        {
            float d[64];
            if (warp < 4) {
                tc::ld_16x256b_x16(tmem + ((uint32_t)(32 * warp) << 16) + COL_W, d);
                tc::wait_ld();
#pragma unroll
                for (int nt = 0; nt < 16; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[0][nt][e] += d[4 * nt + e];
                store_tile_bf16<16, D>(acc, U16, 16 * warp, lane, 1.f);
            } else if (with_o) {
                tc::ld_16x256b_x16(tmem + ((uint32_t)(32 * p) << 16) + COL_Q, d);
                tc::wait_ld();
#pragma unroll
                for (int nt = 0; nt < 16; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[0][nt][e] = d[4 * nt + e];
            }
        }
        if (tid == 0) tc::bulk_wait_read();  // the previous state image is out: S16 may be rewritten below
        tc::fence_async_smem();
        tc::fence_before();
        __syncthreads();
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
        }
        // ---- S += Kh^T U in TMEM
        if (tid == 0) {
            tc::fence_after();
            const uint32_t sK = tc::smem_addr(st.la), sU = tc::smem_addr(U16);
#pragma unroll
            for (int s = 0; s < 4; ++s)
                tc::mma_bf16(tmem + COL_S, tc::sdesc(sK + s * 2048, 8192, 1024), tc::sdesc(sU + s * 2048, 8192, 1024),
                             IDESC_S, true);
            tc::commit(&sm.mbar[1]);
        }
        // ---- O += M U (warps 4..7), store o
        if (warp >= 4 && with_o) {
            warp_gemm<1, 16, true, false, 64, D>(acc, M16, 16 * p, U16, 0, C, lane);
            const int rl = 16 * p + (lane >> 2);
            bf16 *o = static_cast<bf16 *>(a.o);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int t = n * C + rl + 8 * half;
                if (t < a.T) {
                    bf16 *orow = o + (((size_t)b * a.T + t) * a.H + h) * D;
#pragma unroll
                    for (int nt = 0; nt < 16; ++nt)
                        *reinterpret_cast<uint32_t *>(orow + 8 * nt + 2 * (lane & 3)) =
                            pack_bf16(acc[0][nt][2 * half], acc[0][nt][2 * half + 1]);
                }
            }
        }
        if (!tc::mbar_wait(&sm.mbar[1], ph1)) {
            sm.abort = 1;
            record_status(a.status, GDN2_ERR_TIMEOUT);
        }
        ph1 ^= 1;
        tc::fence_after();

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
