// Gate-aware backward (vector-Jacobian product) of the chunk-parallel forward.
//
// "Why NVIDIA Gated DeltaNet-2 separates erase and write gates" (axbrief),
// section "Gated Delta Rule-2: per-channel erase/write split": the backward
// can no longer use KDA's scalar shortcut, because the distinct diagonal
// gates on the erase side (b, key axis) and the write side (w, value axis)
// sit inside every gradient-accumulating inner product.  Here b enters through
// g = b . k inside the key Gram and the erase term, and w through w . v in
// the value targets; their gradients are taken inside those products.
//
// Two launches.  (1) Unless the training forward already kept them, the
// forward kernel re-runs and writes the bf16 state at every chunk boundary and
// each chunk's T, M and U tiles to the workspace.  (2) The reverse pass walks
// each (batch, head) sequence's chunks in reverse order, carrying
// dSigma = dL/dS(chunk end) in fp32.  This file's kernel does it with
// warp-level products for every head size; dk = dv = 128 goes to the
// tensor-memory kernel of chunk_bwd_tc.cu.  For a chunk with start state S,
// end state Sigma and the forward's quantities (chunk_common.cuh, fast path;
// Dh = Diag(gam) dSigma):
//
//   dU   = M^T dO + Kb Dh                    dM = strict_lower(dO U^T), diag(dO U^T)
//   nR   = -T^T dU      (= -dRHS)            dA = strict_lower(nR U^T)
//   dv   = -nR . w,  dw = -nR . v (bf16 nR)  dKb = U Dh^T + dA^T Gt + dM^T Qt
//   dQt  = dO S^T + dM Kb                    dGt = nR S^T + dA Kb
//   dS   = Dh + Qt^T dO + Gt^T nR            (-> dSigma of the previous chunk)
//   dq = dQt e^{L} + dMd k,  dg = dGt e^{L},  dk = dKb e^{-L} + dMd q + dg . b,
//   db = dg . k   (dMd = diagonal of dO U^T)
//   dL_r = dQt.Qt + dGt.Gt - dKb.Kb (+ rowsum(dSigma . Sigma) at the chunk end)
//   dlog_alpha = reverse cumulative sum of dL within the chunk.
//
// A slow chunk (decay beyond e^{-64} inside the chunk) uses Kt = k e^{L_end-L}
// with Dh = dSigma, and takes the Gram gradients term by term in fp32.
//
// dQt, dGt and dKb are staged in fp32 in shared-memory regions that are dead by
// then; the per-CTA fp32 scratch of the caller's workspace (L2-resident) holds
// the slow-path partial gradients and a few row sums.
#include "chunk_bwd_common.cuh"
#include "gdn2.h"

namespace gdn2 {
namespace cbwd {

using namespace chunk;

template <int DK, int DV>
__global__ void __launch_bounds__(NTHR, 1) chunk_bwd_kernel(ChunkBwdArgs a) {
    constexpr int WR = DK / 4, WC = DV / 2;
    constexpr int MTS = WR / 16, NTS = WC / 8;
    constexpr int NTV = DV / 8, NTK = DK / 8;

    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ IntraShared<DK> sh;
    __shared__ float s_dpart[NTHR / (DK / 2)][DK];
    __shared__ float s_dmd[C];
    __shared__ float s_rs[2][DK];
    BwdChunk<DK, DV> x(a, smem, &sh, s_dpart, s_dmd, s_rs);
    const int warp = x.warp, lane = x.lane, bh = blockIdx.x;
    if (!x.sv.ok) {  // packed-sequence offsets out of range: nothing of this sequence is touched
        if (x.tid == 0) record_status(a.status, GDN2_ERR_INVALID_ARG);
        return;
    }
    const int T = x.len, nchunks = x.nchunks;
    const ChunkTiles st = x.st;
    bf16 *dO16 = x.dO16, *S16 = x.S16, *D16 = x.D16, *T16 = x.T16, *M16 = x.M16, *dU16 = x.dU16, *U16 = x.U16;
    bf16 *nR16 = x.nR16, *dM16 = x.dM16, *dA16 = x.dA16;
    // dM's entries reach tens: its products take it as two bf16 tiles, the
    // rounding dM16 and the remainder dMlo16 (about 16 significant bits)
    bf16 *dMlo16 = reinterpret_cast<bf16 *>(smem + BSmem<DK, DV>::OMLO);
    x.dMlo16 = dMlo16;
    float *A32 = x.A32, *T32 = x.T32, *LAM = x.LAM, *DQT = x.DQT, *DGT = x.DGT, *DKB = x.DKB;
    const bf16 *states = x.states;

    // dSigma: fp32, same register tiling as the forward's state
    const int c0 = (warp >> 1) * WR, j0 = (warp & 1) * WC;
    float dS[MTS][NTS][4];
#pragma unroll
    for (int mt = 0; mt < MTS; ++mt)
#pragma unroll
        for (int nt = 0; nt < NTS; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int c = c0 + 16 * mt + (lane >> 2) + (e >> 1) * 8;
                const int j = j0 + 8 * nt + 2 * (lane & 3) + (e & 1);
                dS[mt][nt][e] = a.dS_T ? a.dS_T[(size_t)bh * DK * DV + (size_t)c * DV + j] : 0.f;
            }

    for (int n = nchunks - 1; n >= 0; --n) {
        const int Cn = min(C, T - n * C);
        x.load(n);

        const bool slow = intra_chunk<DK, DV>(st, A32, T32, view(sh), LAM, false, /*prep_only=*/true);

        // ---- Dh = gam . dSigma (fast) or dSigma (slow) as bf16; row sums of
        // dSigma . Sigma (Sigma = next chunk-boundary state) for dL_end
        {
            const bf16 *Snext = states + (size_t)(n + 1) * DK * DV;
#pragma unroll
            for (int mt = 0; mt < MTS; ++mt) {
                const int c = c0 + 16 * mt + (lane >> 2);
                const float g0 = slow ? 1.f : sh.gamma[c], g1 = slow ? 1.f : sh.gamma[c + 8];
                float r0 = 0.f, r1 = 0.f;
#pragma unroll
                for (int nt = 0; nt < NTS; ++nt) {
                    const int j = j0 + 8 * nt + 2 * (lane & 3);
                    *reinterpret_cast<uint32_t *>(D16 + swz<DV, DK>(c, j)) =
                        pack_bf16(g0 * dS[mt][nt][0], g0 * dS[mt][nt][1]);
                    *reinterpret_cast<uint32_t *>(D16 + swz<DV, DK>(c + 8, j)) =
                        pack_bf16(g1 * dS[mt][nt][2], g1 * dS[mt][nt][3]);
                    const __nv_bfloat162 s0 = *reinterpret_cast<const __nv_bfloat162 *>(Snext + (size_t)c * DV + j);
                    const __nv_bfloat162 s1 =
                        *reinterpret_cast<const __nv_bfloat162 *>(Snext + (size_t)(c + 8) * DV + j);
                    r0 += dS[mt][nt][0] * __low2float(s0) + dS[mt][nt][1] * __high2float(s0);
                    r1 += dS[mt][nt][2] * __low2float(s1) + dS[mt][nt][3] * __high2float(s1);
                }
                r0 += __shfl_xor_sync(0xffffffffu, r0, 1);
                r0 += __shfl_xor_sync(0xffffffffu, r0, 2);
                r1 += __shfl_xor_sync(0xffffffffu, r1, 1);
                r1 += __shfl_xor_sync(0xffffffffu, r1, 2);
                if ((lane & 3) == 0) {
                    s_rs[warp & 1][c] = r0;
                    s_rs[warp & 1][c + 8] = r1;
                }
            }
        }

        constexpr int NTX = NTV > NTK ? NTV : NTK;
        float accX[1][NTX][4];
        auto &accV = reinterpret_cast<float(&)[1][NTV][4]>(accX);
        auto &accK = reinterpret_cast<float(&)[1][NTK][4]>(accX);
        __syncthreads();  // D16 and the row sums are complete

        // ---- dU = M^T dO + Kh Dh (warps 0..3) ; dM = lower(dO U^T) (warps 4..7)
        if (warp < 4) {
            zero(accX);
            warp_gemm<1, NTV, false, false, 64, DV, C, C, KU>(accV, M16, 16 * warp, dO16, 0, C, lane);
            warp_gemm<1, NTV, true, false, DK, DV, C, DK, KU>(accV, st.la, 16 * warp, D16, 0, DK, lane);
            store_tile_bf16<NTV, DV>(accV, dU16, 16 * warp, lane, 1.f);
        } else {
            float acc[1][8][4];
            zero(acc);
            warp_gemm<1, 8, true, true, DV, DV, C, C, KU>(acc, dO16, 16 * (warp & 3), U16, 0, DV, lane);
            const int r0 = 16 * (warp & 3) + (lane >> 2);
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    // The diagonal of M carries no decay factor (e^{L_r - L_r} = 1):
                    // its gradient goes straight to dq and dk in fp32 and is kept
                    // out of the Gram products, where it would cancel in dL.
                    const int r = r0 + (e >> 1) * 8, i = 8 * nt + 2 * (lane & 3) + (e & 1);
                    if (i == r) s_dmd[r] = acc[0][nt][e];
                    if (i >= r) acc[0][nt][e] = 0.f;
                }
            store_tile_bf16<8, 64>(acc, dM16, 16 * (warp & 3), lane, 1.f);
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    acc[0][nt][e] -= __bfloat162float(__float2bfloat16_rn(acc[0][nt][e]));
            store_tile_bf16<8, 64>(acc, dMlo16, 16 * (warp & 3), lane, 1.f);
        }
        __syncthreads();

        // ---- nR = -T^T dU (warps 0..3)
        if (warp < 4) {
            zero(accX);
            warp_gemm<1, NTV, false, false, 64, DV, C, C, KU>(accV, T16, 16 * warp, dU16, 0, C, lane);
            store_tile_bf16<NTV, DV>(accV, nR16, 16 * warp, lane, -1.f);
        }
        __syncthreads();

        // ---- dA = strict_lower(nR U^T) (warps 0..3) ; dQt = dO S^T (warps 4..7)
        if (warp < 4) {
            float acc[1][8][4];
            zero(acc);
            warp_gemm<1, 8, true, true, DV, DV, C, C, KU>(acc, nR16, 16 * warp, U16, 0, DV, lane);
            const int r0 = 16 * warp + (lane >> 2);
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = r0 + (e >> 1) * 8, i = 8 * nt + 2 * (lane & 3) + (e & 1);
                    if (i >= r) acc[0][nt][e] = 0.f;
                }
            store_tile_bf16<8, 64>(acc, dA16, 16 * warp, lane, 1.f);
        } else {
            zero(accX);
            warp_gemm<1, NTK, true, true, DV, DV, C, DK, KU>(accK, dO16, 16 * (warp & 3), S16, 0, DV, lane);
        }
        __syncthreads();

        // ---- dGt = nR S^T + dA Kb (warps 0..3) ; dQt += dM Kb (warps 4..7)
        if (warp < 4) {
            zero(accX);
            warp_gemm<1, NTK, true, true, DV, DV, C, DK, KU>(accK, nR16, 16 * warp, S16, 0, DV, lane);
            if (!slow) warp_gemm<1, NTK, true, false, 64, DK, C, C, KU>(accK, dA16, 16 * warp, st.la, 0, C, lane);
            store_stage<DK, NTK>(accK, DGT, 16 * warp, 0, lane);  // the WY-solve area is dead
        } else if (!slow) {
            warp_gemm<1, NTK, true, false, 64, DK, C, C, KU>(accK, dM16, 16 * (warp & 3), st.la, 0, C, lane);
            warp_gemm<1, NTK, true, false, 64, DK, C, C, KU>(accK, dMlo16, 16 * (warp & 3), st.la, 0, C, lane);
        }
        __syncthreads();  // S is no longer read: its region takes dQt

        // ---- dKb = U Dh^T + dA^T Gt + dM^T Qt (warps 4..7), then dSigma (all warps)
        if (warp >= 4) {
            const int m0 = 16 * (warp & 3);
            store_stage<DK, NTK>(accK, DQT, m0, 0, lane);
            zero(accX);
            warp_gemm<1, NTK, true, true, DV, DV, C, DK, KU>(accK, U16, m0, D16, 0, DV, lane);
            if (!slow) {
                warp_gemm<1, NTK, false, false, 64, DK, C, C, KU>(accK, dA16, m0, st.b, 0, C, lane);
                warp_gemm<1, NTK, false, false, 64, DK, C, C, KU>(accK, dM16, m0, st.q, 0, C, lane);
                warp_gemm<1, NTK, false, false, 64, DK, C, C, KU>(accK, dMlo16, m0, st.q, 0, C, lane);
            }
            asm volatile("bar.sync 1, 128;\n" ::: "memory");  // warps 4..7 are done reading Dh
            store_stage<DK, NTK>(accK, DKB, m0, 0, lane);
        }

        // ---- dSigma <- Diag(gam) dSigma + Qt^T dO + Gt^T nR (all warps)
#pragma unroll
        for (int mt = 0; mt < MTS; ++mt) {
            const float g0 = sh.gamma[c0 + 16 * mt + (lane >> 2)], g1 = sh.gamma[c0 + 16 * mt + (lane >> 2) + 8];
#pragma unroll
            for (int nt = 0; nt < NTS; ++nt) {
                dS[mt][nt][0] *= g0; dS[mt][nt][1] *= g0; dS[mt][nt][2] *= g1; dS[mt][nt][3] *= g1;
            }
        }
        warp_gemm<MTS, NTS, false, false, DK, DV, C, C, KU>(dS, st.q, c0, dO16, j0, C, lane);
        warp_gemm<MTS, NTS, false, false, DK, DV, C, C, KU>(dS, st.b, c0, nR16, j0, C, lane);
        __syncthreads();

        if (slow) x.slow_grams(n, Cn);
        x.token_grads(n, Cn, slow);
        __syncthreads();
    }

    if (a.dS0) {
#pragma unroll
        for (int mt = 0; mt < MTS; ++mt)
#pragma unroll
            for (int nt = 0; nt < NTS; ++nt)
#pragma unroll
                for (int e = 0; e < 4; e += 2) {
                    const int c = c0 + 16 * mt + (lane >> 2) + (e >> 1) * 8;
                    const int j = j0 + 8 * nt + 2 * (lane & 3);
                    *reinterpret_cast<float2 *>(a.dS0 + (size_t)bh * DK * DV + (size_t)c * DV + j) =
                        make_float2(dS[mt][nt][e], dS[mt][nt][e + 1]);
                }
    }
}

template <int DK, int DV>
cudaError_t launch_t(const ChunkBwdArgs &a, cudaStream_t s) {
    // (1) state pass: the forward with bf16 chunk-boundary states, no output
    // (skipped when the forward already saved them)
    cudaError_t e = cudaSuccess;
    if (!a.states_given) {
        ChunkFwdArgs f{a.q, a.k, a.v, a.log_alpha, a.b, a.w, a.S0, nullptr, nullptr, a.scratch, a.scr_stride,
                       a.states, a.intra, a.ops, a.status, a.B, a.T, a.H, a.cu_seqlens};
        f.gates = a.gates;
        e = launch_chunk_fwd(f, DK, DV, s);
        if (e != cudaSuccess) return e;
    }
    // (2) reverse chunk pass (tensor-memory products for dk = dv = 128)
    if constexpr (DK == 128 && DV == 128) {
        return launch_chunk_bwd_tc(a, s);
    } else {
        constexpr int bytes = BSmem<DK, DV>::BYTES;
        e = cudaFuncSetAttribute(chunk_bwd_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e != cudaSuccess) return e;
        chunk_bwd_kernel<DK, DV><<<(unsigned)(a.B * a.H), NTHR, bytes, s>>>(a);
        return cudaGetLastError();
    }
}

template <int DK, int DV>
size_t ws_t(int B, int T, int H, size_t *scr_stride, size_t *states_bytes, bool varlen) {
    const size_t sb = states_region_bytes(B, T, H, DK, DV, varlen) + intra_region_bytes(B, T, H, DV, varlen) +
                      ops_region_bytes(B, T, H, DK, DV, varlen);
    const size_t stride = (Scratch<DK>::FLOATS + 63) / 64 * 64;
    if (scr_stride) *scr_stride = stride;
    if (states_bytes) *states_bytes = sb;
    return sb + (size_t)B * H * stride * sizeof(float);
}

}  // namespace cbwd

size_t chunk_bwd_ws_bytes(int B, int T, int H, int dk, int dv, size_t *scr_stride, size_t *states_bytes,
                          bool varlen) {
    if (dk == 128 && dv == 128) return cbwd::ws_t<128, 128>(B, T, H, scr_stride, states_bytes, varlen);
    if (dk == 128 && dv == 64) return cbwd::ws_t<128, 64>(B, T, H, scr_stride, states_bytes, varlen);
    if (dk == 64 && dv == 128) return cbwd::ws_t<64, 128>(B, T, H, scr_stride, states_bytes, varlen);
    return cbwd::ws_t<64, 64>(B, T, H, scr_stride, states_bytes, varlen);
}

cudaError_t launch_chunk_bwd(const ChunkBwdArgs &a, int dk, int dv, cudaStream_t s) {
    if (dk == 128 && dv == 128) return cbwd::launch_t<128, 128>(a, s);
    if (dk == 128 && dv == 64) return cbwd::launch_t<128, 64>(a, s);
    if (dk == 64 && dv == 128) return cbwd::launch_t<64, 128>(a, s);
    return cbwd::launch_t<64, 64>(a, s);
}

}  // namespace gdn2
