// tcgen05 operands and results on the swizzled shared-memory tiles of
// chunk_common.cuh (64-column blocks of 128-byte rows, 16-byte chunks permuted
// by row mod 8 — the 128-byte-swizzle canonical layout): operand descriptors,
// an MMA group over K, and the 16x256b tensor-memory fragments that land in
// the register layout of a warp-level m16n8 product.
#pragma once

#include "chunk_common.cuh"
#include "tc.cuh"

namespace gdn2 {
namespace tct {

using namespace chunk;

// Byte offset of k-step s (16 elements) from k-step 0 of an operand in an
// [R][.] tile: K-major (rows = M or N, columns = K; four k-steps per 128-byte
// swizzle row, then the next 64-column block R * 128 bytes on) or MN-major
// (rows = K: 16 rows of 128 bytes per k-step).
template <bool K_MAJOR>
__host__ __device__ __forceinline__ uint32_t kstep_bytes(int R, int s) {
    return K_MAJOR ? (uint32_t)((s >> 2) * (R * 128) + (s & 3) * 32) : (uint32_t)(s * 2048);
}
// Descriptor of k-step s of such an operand whose tile starts at shared
// address `start`: K-major atoms of 8 rows x 128 bytes stacked every 1024
// bytes along M/N; MN-major atoms of 64 elements x 8 rows, the next 64
// elements R * 128 bytes on, the next 8 K rows 1024 bytes on.
template <bool K_MAJOR>
__host__ __device__ __forceinline__ uint64_t operand_desc(uint32_t start, int R, int s) {
    return K_MAJOR ? tc::sdesc(start + kstep_bytes<true>(R, s), 16, 1024)
                   : tc::sdesc(start + kstep_bytes<false>(R, s), (uint32_t)(R * 128), 1024);
}
__device__ __forceinline__ uint64_t kmaj(const void *tile, int R, int s) {
    return operand_desc<true>(tc::smem_addr(tile), R, s);
}
__device__ __forceinline__ uint64_t mnmaj(const void *tile, int R, int s) {
    return operand_desc<false>(tc::smem_addr(tile), R, s);
}

// D (+)= A B over K = 16 ks, issued by one thread.  A_K / B_K: K-major operand.
// The descriptors of k-step 0 are built once; a later k-step adds its byte
// offset / 16 to the start-address field, which cannot carry out of it
// (shared memory addresses stay below 2^18).
template <bool A_K, bool B_K>
__device__ __forceinline__ void mma_tiles(uint32_t d, const void *A, int RA, const void *B, int RB, int ks,
                                          uint32_t idesc, bool accumulate) {
    const uint64_t da0 = A_K ? kmaj(A, RA, 0) : mnmaj(A, RA, 0);
    const uint64_t db0 = B_K ? kmaj(B, RB, 0) : mnmaj(B, RB, 0);
#pragma unroll
    for (int s = 0; s < ks; ++s)
        tc::mma_bf16(d, da0 + (kstep_bytes<A_K>(RA, s) >> 4), db0 + (kstep_bytes<B_K>(RB, s) >> 4), idesc,
                     accumulate || s > 0);
}

// A fragment of 8 NTL columns of a 64-row accumulator (16 rows per warp),
// read with the 16x256b shape, as a warp-level [1][NTL][4] tile.
template <int NTL>
using Frag = float[1][NTL][4];
__device__ __forceinline__ void ld_frag(uint32_t taddr, Frag<4> &f) {
    tc::ld_16x256b_x4(taddr, reinterpret_cast<float(&)[16]>(f));
}
__device__ __forceinline__ void ld_frag(uint32_t taddr, Frag<8> &f) {
    tc::ld_16x256b_x8(taddr, reinterpret_cast<float(&)[32]>(f));
}

// bf16 store of a fragment (rows m0.., columns n0..) into a swizzled [.][DC] tile.
template <int DC, int NTL>
__device__ __forceinline__ void store_frag_bf16(const Frag<NTL> &f, bf16 *dst, int m0, int n0, int lane,
                                                float scale) {
    const int r = m0 + (lane >> 2);
#pragma unroll
    for (int nt = 0; nt < NTL; ++nt) {
        const int c = n0 + 8 * nt + 2 * (lane & 3);
        *reinterpret_cast<uint32_t *>(dst + swz<DC>(r, c)) = pack_bf16(scale * f[0][nt][0], scale * f[0][nt][1]);
        *reinterpret_cast<uint32_t *>(dst + swz<DC>(r + 8, c)) = pack_bf16(scale * f[0][nt][2], scale * f[0][nt][3]);
    }
}

// sum_e v[e] * y[e] over 8 fp32 values and 8 packed bf16 values
// (pairs on the packed fp32x2 pipe)
__device__ __forceinline__ float dot8(const float *v, uint4 y) {
    const __nv_bfloat162 *y2 = reinterpret_cast<const __nv_bfloat162 *>(&y);
    float2 acc = __fmul2_rn(make_float2(v[0], v[1]), __bfloat1622float2(y2[0]));
#pragma unroll
    for (int e = 1; e < 4; ++e) acc = __ffma2_rn(make_float2(v[2 * e], v[2 * e + 1]), __bfloat1622float2(y2[e]), acc);
    return acc.x + acc.y;
}

}  // namespace tct
}  // namespace gdn2
