// Building blocks shared by the chunk-parallel forward and backward kernels:
// warp-level bf16 tensor-core products over swizzled shared-memory tiles,
// cp.async tile loads, and the intra-chunk stage (decay prefix, gated and
// decay-referenced operands, key Gram matrices, the WY solve).
//
// Chunk algebra ("Why NVIDIA Gated DeltaNet-2 separates erase and write
// gates", section "Gated Delta Rule-2: per-channel erase/write split"; WY form
// from the laonpeople Gated DeltaNet page, parallel-computation section).  For
// a chunk of C = 64 tokens, L = in-chunk cumulative log-decay, g = b . k:
//
//   Gt = g e^{L}, Qt = q e^{L}  (in (0,1]),   Kb = k e^{-L},   gam = e^{L_end}
//   A = strict_lower([Gt] Kb^T),  M = lower([Qt] Kb^T),  T = (I + A)^{-1}
//
// Kb grows with the decay inside the chunk.  A chunk in which a key channel
// decays by more than e^{-64} ("slow" chunk) forms A and M term by term from
// e^{L_r - L_i} <= 1 instead and replaces Kb by Kt = k e^{L_end - L} (<= 1).
#pragma once

#include "common.cuh"

namespace gdn2 {
namespace chunk {

typedef __nv_bfloat16 bf16;
constexpr int C = 64;
constexpr int NTHR = 256;
constexpr float kSpanGuard = 64.f;  // max in-chunk log-decay span of the fast path

// Shared-memory tiles of R rows x D bf16 columns are stored as D/64 blocks of
// [R][64] (128-byte rows); within a block the 16-byte chunk index of row r is
// XORed with (r & 7).  This is the 128-byte-swizzled canonical layout of the
// tensor-core operand descriptors (8-row x 128-byte atoms, K-major when rows
// are the M/N index, MN-major when rows are the K index), and it keeps
// ldmatrix row addresses in distinct banks.  Tiles start on 1 KB boundaries.
template <int D, int R = 64>
__device__ __forceinline__ int swz(int r, int c) {
    static_assert(D == 64 || D == 128, "tile width");
    return (c >> 6) * (R * 64) + r * 64 + ((((c >> 3) & 7) ^ (r & 7)) << 3) + (c & 7);
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
// the two bf16 values packed in x (the low half first) as fp32
__device__ __forceinline__ float2 unpack_bf16(uint32_t x) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&x));
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool ok) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(ok ? 16 : 0));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// acc[MT][NT][4] += A[m0 + 16 mt + .., k] * B[k, n0 + 8 nt + ..], k in [0, K).
// A_KM: A stored [m][k] in a [RA][DA] tile, else stored [k][m].
// B_KM: B stored [n][k] in a [RB][DB] tile, else stored [k][n].
// One k-step of 16 of warp_gemm below.
template <int MT, int NT, bool A_KM, bool B_KM, int DA, int DB, int RA, int RB>
__device__ __forceinline__ void warp_gemm_kstep(float (&acc)[MT][NT][4], const bf16 *A, int m0, const bf16 *B,
                                                int n0, int k0, int lane) {
    uint32_t a[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        if (A_KM) {
            const int r = m0 + 16 * mt + (lane & 7) + ((lane >> 3) & 1) * 8;
            const int c = k0 + (lane >> 4) * 8;
            ldsm4(smem_u32(A + swz<DA, RA>(r, c)), a[mt]);
        } else {
            const int i = lane >> 3;
            const int kr = k0 + (lane & 7) + (i >> 1) * 8;
            const int mc = m0 + 16 * mt + (i & 1) * 8;
            ldsm4t(smem_u32(A + swz<DA, RA>(kr, mc)), a[mt]);
        }
    }
#pragma unroll
    for (int np = 0; np < NT / 2; ++np) {
        uint32_t b[4];
        if (B_KM) {
            const int r = n0 + 16 * np + (lane & 7) + (lane >> 4) * 8;
            const int c = k0 + ((lane >> 3) & 1) * 8;
            ldsm4(smem_u32(B + swz<DB, RB>(r, c)), b);
        } else {
            const int kr = k0 + (lane & 7) + ((lane >> 3) & 1) * 8;
            const int nc = n0 + 16 * np + (lane >> 4) * 8;
            ldsm4t(smem_u32(B + swz<DB, RB>(kr, nc)), b);
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            mma16816(acc[mt][2 * np], a[mt], b[0], b[1]);
            mma16816(acc[mt][2 * np + 1], a[mt], b[2], b[3]);
        }
    }
}

// acc[MT][NT][4] += A[m0 + 16 mt + .., k] * B[k, n0 + 8 nt + ..], k in [0, K).
// A_KM: A stored [m][k] in a [RA][DA] tile, else stored [k][m].
// B_KM: B stored [n][k] in a [RB][DB] tile, else stored [k][n].
// UNR: unroll factor of the k loop (0 = full); a rolled loop keeps long
// straight-line kernels inside the instruction cache.
template <int MT, int NT, bool A_KM, bool B_KM, int DA, int DB, int RA = C, int RB = C, int UNR = 0>
__device__ __forceinline__ void warp_gemm(float (&acc)[MT][NT][4], const bf16 *A, int m0, const bf16 *B,
                                          int n0, int K, int lane) {
    static_assert(NT % 2 == 0, "n tiles come in pairs");
    if constexpr (UNR == 0) {
#pragma unroll
        for (int k0 = 0; k0 < K; k0 += 16)
            warp_gemm_kstep<MT, NT, A_KM, B_KM, DA, DB, RA, RB>(acc, A, m0, B, n0, k0, lane);
    } else {
#pragma unroll UNR
        for (int k0 = 0; k0 < K; k0 += 16)
            warp_gemm_kstep<MT, NT, A_KM, B_KM, DA, DB, RA, RB>(acc, A, m0, B, n0, k0, lane);
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

// cp.async of tokens [n*C, n*C + C) of one sequence (head h; its tokens are
// the rows row0 .. row0 + len - 1 of a token tensor [rows][H][D]) into a
// swizzled [C][D] tile; tokens past len are zero-filled.
template <int D, int NT = NTHR>
__device__ __forceinline__ void load_token_tile(bf16 *dst, const bf16 *src, size_t row0, int len, int h, int n,
                                                int H) {
    constexpr int CPR = D / 8;  // 16-byte chunks per row
    for (int id = threadIdx.x; id < C * CPR; id += NT) {
        const int r = id / CPR, ch = id % CPR;
        const int t = n * C + r;
        const bool ok = t < len;
        const bf16 *g = src + (ok ? (((row0 + t) * H + h) * D + ch * 8) : 0);
        cp_async16(dst + swz<D>(r, ch * 8), g, ok);
    }
}

// L2 prefetch (no shared-memory destination) of tokens [n*C, n*C + C) of one
// sequence (rows row0 .. of a token tensor [rows][H][D]), one bulk request per
// row; thread `slot` of `nslots`.
template <int D>
__device__ __forceinline__ void prefetch_token_rows_l2(const bf16 *src, size_t row0, int len, int h, int n, int H,
                                                       int slot, int nslots) {
    for (int r = slot; r < C; r += nslots) {
        const int t = n * C + r;
        if (t < len) {
            const bf16 *g = src + ((row0 + t) * H + h) * D;
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(g), "r"(D * 2) : "memory");
        }
    }
}

// Block-wide 16-byte copy of `bytes` (a multiple of 16) from shared to global memory.
__device__ __forceinline__ void copy_smem_to_global(void *dst, const void *src, int bytes) {
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
    for (int i = threadIdx.x; i < bytes / 16; i += NTHR) d4[i] = s4[i];
}

struct ChunkTiles {
    bf16 *q, *k, *la, *b, *v, *w;
};

// Shared-memory scratch of the intra-chunk stage (static, per CTA of NT threads).
template <int DK, int NT = NTHR>
struct IntraShared {
    float part[NT / (DK / 2)][DK];  // segment sums of log_alpha (channel-pair layout)
    float gamma[DK];
    int slow;
};
// Where the intra-chunk stage keeps that scratch (which may be split).
template <int DK>
struct IntraView {
    float (*part)[DK];
    float *gamma;
    int *slow;
};
template <int DK, int NT>
__device__ __forceinline__ IntraView<DK> view(IntraShared<DK, NT> &s) {
    return {s.part, s.gamma, &s.slow};
}

// The threads that run a stage: the whole CTA (BAR = 0, __syncthreads), or
// the NT threads from thread BASE on, which meet at the named barrier BAR.
template <int BAR, int NT, int BASE>
struct Grp {
    static __device__ __forceinline__ void sync() {
        if constexpr (BAR == 0) __syncthreads();
        else asm volatile("bar.sync %0, %1;\n" ::"n"(BAR), "n"(NT) : "memory");
    }
    static __device__ __forceinline__ int tid() { return (int)threadIdx.x - BASE; }
};

// The fp32 [64][64] work arrays of the WY solve (A, T) are row-major with the
// 16-byte column group of row r XORed with r & 7: the eight rows that one
// access of a warp touches (a TF32 A fragment, a fragment write-back) then lie
// in distinct banks instead of all in the same four.
__device__ __forceinline__ int fsw(int r, int c) { return r * C + (c ^ ((r & 7) << 2)); }

// TF32 operand from fp32 bits: the tensor cores read the sign, the exponent and
// the top 10 mantissa bits, so adding half a unit of the 10th bit (2^12 to the
// bit pattern) rounds the magnitude to nearest with ties away from zero (a
// carry into the exponent is the correct rounding up a binade), with one
// integer add instead of a conversion.
__device__ __forceinline__ uint32_t tf32_round(uint32_t bits) { return bits + 0x1000u; }
__device__ __forceinline__ uint32_t to_tf32(float x) { return tf32_round(__float_as_uint(x)); }
__device__ __forceinline__ void mma1688_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// One 16x16 block product on the tensor cores in TF32, operands read from
// fp32 [64][64] work arrays (fsw layout): acc += X[r0.., k0..k0+16) * Y[k0.., c0..c0+16).
__device__ __forceinline__ void block16_tf32(float (&acc)[2][4], const float *X, int r0, int k0, const float *Y,
                                             int c0, int lane) {
    const int g = lane >> 2, t = lane & 3;
    // A fragments by ldmatrix (four 8-row x 16-byte matrices of 32-bit words):
    // lane l addresses row r0 + (l & 7) + 8 ((l >> 3) & 1) at column group
    // (l >> 4) of the k-step; fsw keeps each 16-byte group whole
    const int lr = r0 + (lane & 7) + 8 * ((lane >> 3) & 1), lc = 4 * (lane >> 4);
#pragma unroll
    for (int kk = 0; kk < 16; kk += 8) {
        uint32_t a[4];
        ldsm4(smem_u32(X + fsw(lr, k0 + kk + lc)), a);
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = tf32_round(a[i]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const uint32_t b0 = to_tf32(Y[fsw(k0 + kk + t, c0 + 8 * nt + g)]);
            const uint32_t b1 = to_tf32(Y[fsw(k0 + kk + t + 4, c0 + 8 * nt + g)]);
            mma1688_tf32(acc[nt], a, b0, b1);
        }
    }
}

// Column j of the inverse of the unit lower-triangular 16x16 diagonal block R
// of I + A (A: fp32 [64][64], fsw layout), row by row: x_s = [s == j] -
// sum_{r < s} A[s][r] x_r.  Row s of the block is read as 16-byte groups
// (rows 16 R + s have r & 7 = s & 7, so column group q of the block sits at
// (16 R + 4 q) ^ 4 (s & 7)), the same address for all 16 threads of a block.
__device__ __forceinline__ void diag_column(const float *A32, int R, int j, float (&x)[16]) {
#pragma unroll
    for (int s = 0; s < 16; ++s) {
        const float *row = A32 + (16 * R + s) * C;
        float acc = s == j ? 1.f : 0.f;
#pragma unroll
        for (int q = 0; 4 * q < s; ++q) {
            const float4 a4 = *reinterpret_cast<const float4 *>(row + ((16 * R + 4 * q) ^ ((s & 7) << 2)));
            const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (4 * q + e < s) acc = fmaf(-av[e], x[4 * q + e], acc);
        }
        x[s] = acc;
    }
}

// The four diagonal-block inverses into Tdiag ([4][16][16] fp32, row-major
// blocks): threads 0..63 of G, one column each; no barrier.
template <class G>
__device__ __forceinline__ void wy_diag(const float *A32, float *Tdiag) {
    const int tid = G::tid();
    if (tid < 64) {
        const int R = tid >> 4, j = tid & 15;
        float x[16];
        diag_column(A32, R, j, x);
#pragma unroll
        for (int r = 0; r < 16; ++r) Tdiag[R * 256 + r * 16 + j] = x[r];
    }
}

// WY solve: T = (I + A)^{-1} for the strictly lower 64x64 A in the fp32 area
// A32 (fsw layout), in the fp32 work area T32 (fsw layout) and then as T16 =
// bf16 T (swizzled [64][64]; T16 may be the first half of the T32 area).  All
// NT threads of G; on return the T32 area past T16 may be written, and T16 is
// complete after the caller's next barrier.  With Tdiag the four diagonal-block
// inverses come ready-made (wy_diag, [4][16][16] fp32); else they are formed here.
template <int NT, class G = Grp<0, NT, 0>>
__device__ void wy_solve(const float *A32, float *T32, bf16 *T16, const float *Tdiag = nullptr) {
    const int tid = G::tid(), warp = tid >> 5, lane = tid & 31;
    // 16x16 diagonal blocks (fp32), the blocks above them zero
    if (Tdiag) {  // (every load before the first store, which would order the later loads)
        static_assert(1024 % NT == 0, "whole blocks");
        constexpr int ND = 1024 / NT;
        float dv[ND];
#pragma unroll
        for (int i = 0; i < ND; ++i) dv[i] = Tdiag[tid + NT * i];
#pragma unroll
        for (int i = 0; i < ND; ++i) {
            const int e = tid + NT * i, blk = e >> 8, r = (e >> 4) & 15, c = e & 15;
            T32[fsw(16 * blk + r, 16 * blk + c)] = dv[i];
        }
        for (int e = tid; e < 6 * 256; e += NT) {
            const int u = e >> 8, r = (e >> 4) & 15, c = e & 15;
            const int R = u < 3 ? 0 : (u < 5 ? 1 : 2), Q = u < 3 ? u + 1 : (u < 5 ? u - 1 : 3);
            T32[fsw(16 * R + r, 16 * Q + c)] = 0.f;
        }
    } else if (tid < 64) {
        const int R = tid >> 4, j = tid & 15;
        float x[16];
        diag_column(A32, R, j, x);
#pragma unroll
        for (int r = 0; r < 16; ++r) T32[fsw(16 * R + r, 16 * R + j)] = x[r];
    } else {
        for (int e = tid - 64; e < 6 * 256; e += NT - 64) {
            const int blk = e >> 8, r = (e >> 4) & 15, c = e & 15;
            const int R = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
            const int Q = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
            T32[fsw(16 * R + r, 16 * Q + c)] = 0.f;
        }
    }
    G::sync();
    // Off-diagonal blocks on the tensor cores in TF32 (T is rounded to bf16
    // afterwards), two levels of 32 x 32 blocks, one warp per 16 x 16 block:
    //   T10 = -T11 A10 T00,  T32 = -T33 A32 T22;
    //   [T20 T21; T30 T31] = -[T22 0; T32 T33] X,  X = A[2:4, 0:2] [T00 0; T10 T11],
    // where X's terms that need no T10 start beside T10 and T32.
    const int g = lane >> 2, t = lane & 3;
    auto put = [&](const float (&x)[2][4], int R, int Q, float sc) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int c = 16 * Q + 8 * nt + 2 * t;
            *reinterpret_cast<float2 *>(T32 + fsw(16 * R + g, c)) = make_float2(sc * x[nt][0], sc * x[nt][1]);
            *reinterpret_cast<float2 *>(T32 + fsw(16 * R + g + 8, c)) = make_float2(sc * x[nt][2], sc * x[nt][3]);
        }
    };
    float x[2][4] = {};
    if (warp < 2) {  // T10 (warp 0) and T32 (warp 1): Z = A_RQ T_QQ, then -T_RR Z
        const int Q = 2 * warp, R = Q + 1;
        block16_tf32(x, A32, 16 * R, 16 * Q, T32, 16 * Q, lane);
        put(x, R, Q, 1.f);
        __syncwarp();
        float y[2][4] = {};
        block16_tf32(y, T32, 16 * R, 16 * R, T32, 16 * Q, lane);
        __syncwarp();
        put(y, R, Q, -1.f);
    } else if (warp < 6) {  // X20, X30 (first terms), X21, X31
        const int R = 2 + (warp & 1), Q = (warp - 2) >> 1;
        block16_tf32(x, A32, 16 * R, 16 * Q, T32, 16 * Q, lane);  // A_R0 T00 or A_R1 T11
    }
    G::sync();
    if (warp >= 2 && warp < 6) {
        const int R = 2 + (warp & 1), Q = (warp - 2) >> 1;
        if (Q == 0) block16_tf32(x, A32, 16 * R, 16, T32, 0, lane);  // + A_R1 T10
        put(x, R, Q, 1.f);                                           // X_RQ in the T_RQ slot
    }
    G::sync();
    if (warp < 4) {  // Y = [T22 0; T32 T33] X into registers, then -Y
        const int R = 2 + (warp >> 1), Q = warp & 1;
        float y[2][4] = {};
        block16_tf32(y, T32, 16 * R, 32, T32, 16 * Q, lane);                 // T_R2 X_2Q
        if (R == 3) block16_tf32(y, T32, 48, 48, T32, 16 * Q, lane);         // + T33 X_3Q
        G::sync();
        put(y, R, Q, -1.f);
    } else {
        G::sync();
    }
    G::sync();
    // T32 -> T16 (bf16, swizzled [64][64], the first half of the T32 area)
    {
        constexpr int EPT = C * C / NT;  // elements per thread (row r, columns cb ..)
        static_assert(EPT % 4 == 0, "whole column groups");
        const int r = tid / (C / EPT), cb = (tid % (C / EPT)) * EPT;
        float tv[EPT];
#pragma unroll
        for (int s = 0; s < EPT; s += 4) {
            const float4 v4 = *reinterpret_cast<const float4 *>(T32 + fsw(r, cb + s));
            tv[s] = v4.x; tv[s + 1] = v4.y; tv[s + 2] = v4.z; tv[s + 3] = v4.w;
        }
        G::sync();
#pragma unroll
        for (int s = 0; s < EPT; s += 2)
            *reinterpret_cast<uint32_t *>(T16 + swz<64>(r, cb + s)) = pack_bf16(tv[s], tv[s + 1]);
    }
}

// w . v in place of v (the NT threads of G; no barrier).
template <int DV, int NT, class G = Grp<0, NT, 0>>
__device__ __forceinline__ void form_wv(ChunkTiles st) {
    for (int id = G::tid(); id < C * DV / 8; id += NT) {
        // the product of two bf16 values is exact in fp32, so the bf16x2 multiply
        // (one rounding) gives the same bits as an fp32 product rounded to bf16
        uint4 wv = reinterpret_cast<const uint4 *>(st.w)[id];
        uint4 vv = reinterpret_cast<const uint4 *>(st.v)[id];
        const __nv_bfloat162 *w2 = reinterpret_cast<const __nv_bfloat162 *>(&wv);
        const __nv_bfloat162 *v2 = reinterpret_cast<const __nv_bfloat162 *>(&vv);
        uint4 o;
        __nv_bfloat162 *o2 = reinterpret_cast<__nv_bfloat162 *>(&o);
#pragma unroll
        for (int e = 0; e < 4; ++e) o2[e] = __hmul2(w2[e], v2[e]);
        reinterpret_cast<uint4 *>(st.v)[id] = o;
    }
}

// Intra-chunk stage.  On entry the six raw token tiles of the chunk are in
// shared memory (and visible to all threads).  With prep_only only the decay
// prefix and the operands Qt, Gt, Kb/Kt are formed (v, w untouched; T, M
// come from elsewhere).  With grams_ext a fast chunk stops there too (the
// caller forms A, M and T); with pass1_only (which implies prep_only) only the
// segment sums, gam and a slow chunk's L are formed (the operands come from
// elsewhere); without wv_here the caller forms w . v (form_wv)
// for a fast chunk, and the slow path forms it before reusing the w tile.
// The scratch's part array needs NT / (DK / 2) - 1 rows.  Otherwise, on exit
// (all threads, after a barrier):
//   st.q -> Qt, st.b -> Gt, st.la -> Kb (fast) or Kt (slow), st.v -> w . v;
//   T16 = bf16 (I + A)^{-1} and M16 = bf16 M (swizzled [64][64]);
//   sh.gamma = e^{L_end}; returns true for a slow chunk.
// A32 and T32 are 64x64 fp32 work areas; A32 is free on return, T32 holds
// T16 and M16.  lam_ws (per-CTA [64][DK] fp32, global) receives L when
// keep_lam is set and is always used by a slow chunk.
// NT: threads of the CTA (a multiple of 64, at least 256).
// G: the threads that run it (the whole CTA by default).
template <int DK, int DV, int NT = NTHR, class G = Grp<0, NT, 0>>
__device__ bool intra_chunk(ChunkTiles st, float *A32, float *T32, IntraView<DK> sh, float *lam_ws,
                            bool keep_lam, bool prep_only = false, bool grams_ext = false, bool wv_here = true,
                            bool pass1_only = false) {
    static_assert(NT % 64 == 0 && NT >= 256, "thread count");
    const int tid = G::tid(), warp = tid >> 5, lane = tid & 31;
    bf16 *M16 = reinterpret_cast<bf16 *>(T32) + C * C;

    if (tid == 0) *sh.slow = 0;
    // ---- pass 1: w . v in place of v (unless the caller forms it later), and the
    // segment sums of log_alpha per channel pair; only the first P2 - 1 are
    // stored (the last segment's threads form the chunk total themselves)
    constexpr int NP = DK / 2, P2 = NT / NP, RS2 = C / P2;
    const int cp = tid % NP, s2 = tid / NP, c2 = 2 * cp;
    if (!prep_only && wv_here) form_wv<DV, NT, G>(st);
    // this thread's rows s2 RS2 .. of its channel pair stay in registers for pass 2
    __nv_bfloat162 la2[RS2];
#pragma unroll
    for (int i = 0; i < RS2; ++i) la2[i] = *reinterpret_cast<const __nv_bfloat162 *>(st.la + swz<DK>(s2 * RS2 + i, c2));
    float2 psum = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < RS2; ++i) psum = __fadd2_rn(psum, __bfloat1622float2(la2[i]));
    const float pa = psum.x, pb = psum.y;
    if (s2 < P2 - 1) {
        sh.part[s2][c2] = pa;
        sh.part[s2][c2 + 1] = pb;
    }
    G::sync();
    float la0 = 0.f, lb0 = 0.f;
#pragma unroll
    for (int s = 0; s < P2 - 1; ++s)
        if (s < s2) { la0 += sh.part[s][c2]; lb0 += sh.part[s][c2 + 1]; }
    if (s2 == P2 - 1) {
        const float la_end = la0 + pa, lb_end = lb0 + pb;
        sh.gamma[c2] = __expf(la_end);
        sh.gamma[c2 + 1] = __expf(lb_end);
        if (-la_end > kSpanGuard || -lb_end > kSpanGuard) *sh.slow = 1;
    }
    G::sync();
    const bool slow = *sh.slow != 0;
    if (pass1_only) {  // the operands come from elsewhere: gam, the segment sums and a slow chunk's L
        if (slow) {
            if (tid < DK) {
                float lam = 0.f;
                for (int r = 0; r < C; ++r) {
                    lam += __bfloat162float(st.la[swz<DK>(r, tid)]);
                    lam_ws[r * DK + tid] = lam;
                }
            }
            G::sync();
        }
        return slow;
    }

    float accM[1][8][4];  // M rows of warps 4..7 (lower incl. diagonal)
    if (!slow) {
        // ---- pass 2 (fast): Qt, Gt, Kb in place of q, b, log_alpha (two channels per thread)
        // (both channels of a thread on the packed fp32x2 pipe)
        // the loads of a batch of the thread's rows are issued before its first
        // store: the in-place stores would otherwise order each row's loads
        // behind the previous row's stores (the tiles are separate arrays, but
        // the compiler cannot tell)
        float2 lam = make_float2(la0, lb0);
        constexpr int RB = RS2 > 8 ? 8 : RS2;  // rows per batch
#pragma unroll
        for (int i0 = 0; i0 < RS2; i0 += RB) {
            __nv_bfloat162 qr[RB], kr[RB], br[RB];
#pragma unroll
            for (int j = 0; j < RB; ++j) {
                const int o = swz<DK>(s2 * RS2 + i0 + j, c2);
                qr[j] = *reinterpret_cast<const __nv_bfloat162 *>(st.q + o);
                kr[j] = *reinterpret_cast<const __nv_bfloat162 *>(st.k + o);
                br[j] = *reinterpret_cast<const __nv_bfloat162 *>(st.b + o);
            }
#pragma unroll
            for (int j = 0; j < RB; ++j) {
                const int i = i0 + j, r = s2 * RS2 + i, o = swz<DK>(r, c2);
                const float2 l = __bfloat1622float2(la2[i]);
                const float2 q2 = __bfloat1622float2(qr[j]);
                const float2 k2 = __bfloat1622float2(kr[j]);
                const float2 b2 = __bfloat1622float2(br[j]);
                lam = __fadd2_rn(lam, l);
                if (keep_lam) *reinterpret_cast<float2 *>(lam_ws + r * DK + c2) = lam;
                const float2 e = make_float2(__expf(lam.x), __expf(lam.y));
                const float2 ie = make_float2(__expf(-lam.x), __expf(-lam.y));
                const float2 qt = __fmul2_rn(q2, e), gt = __fmul2_rn(__fmul2_rn(b2, k2), e), kb = __fmul2_rn(k2, ie);
                *reinterpret_cast<uint32_t *>(st.q + o) = pack_bf16(qt.x, qt.y);
                *reinterpret_cast<uint32_t *>(st.b + o) = pack_bf16(gt.x, gt.y);
                *reinterpret_cast<uint32_t *>(st.la + o) = pack_bf16(kb.x, kb.y);
            }
        }
        G::sync();
        if (prep_only || grams_ext) return false;
        // ---- Grams: [Gt; Qt] Kb^T, warp w < 8 -> rows 16w..16w+15 of the stacked operand
        if (warp < 8) {
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
                    if (warp < 4) A32[fsw(r, i)] = i < r ? acc[0][nt][e] : 0.f;
                    else accM[0][nt][e] = i <= r ? acc[0][nt][e] : 0.f;
                }
        }
    } else {
        // ---- slow chunk: exact per-term decays.  L goes to the per-CTA
        // workspace (one thread per key channel); raw q, k, b stay in shared
        // memory until A and M exist.  w . v is formed first when the caller
        // deferred it: the w tile becomes the T32 work area below.
        if (!prep_only && !wv_here) form_wv<DV, NT, G>(st);
        if (tid < DK) {
            float lam = 0.f;
            for (int r = 0; r < C; ++r) {
                lam += __bfloat162float(st.la[swz<DK>(r, tid)]);
                lam_ws[r * DK + tid] = lam;
            }
        }
        G::sync();
        constexpr int NPAIR = C * (C + 1) / 2, NS = (NPAIR + NT - 1) / NT;
        float pa[NS], pm[NS];
#pragma unroll
        for (int s = 0; s < NS; ++s) {
            pa[s] = 0.f;
            pm[s] = 0.f;
            const int p = tid + NT * s;
            if (!prep_only && p < C * (C + 1) / 2) {
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
        G::sync();
        // Qt, Gt and Kt = k e^{L_end - L} in place of q, b, log_alpha
        if (tid < DK) {
            const float lend = lam_ws[(C - 1) * DK + tid];
            for (int r = 0; r < C; ++r) {
                const int o = swz<DK>(r, tid);
                const float lr = lam_ws[r * DK + tid];
                const float e = __expf(lr);
                const float kk = __bfloat162float(st.k[o]);
                st.q[o] = __float2bfloat16_rn(__bfloat162float(st.q[o]) * e);
                st.b[o] = __float2bfloat16_rn(__bfloat162float(st.b[o]) * kk * e);
                st.la[o] = __float2bfloat16_rn(kk * __expf(lend - lr));
            }
        }
        G::sync();
        if (prep_only) return true;
        for (int e = tid; e < C * C; e += NT) {
            A32[e] = 0.f;
            T32[e] = 0.f;
        }
        G::sync();
#pragma unroll
        for (int s = 0; s < NS; ++s) {
            const int p = tid + NT * s;
            if (p < C * (C + 1) / 2) {
                int r = (int)((sqrtf(8.f * p + 1.f) - 1.f) * 0.5f);
                while ((r + 1) * (r + 2) / 2 <= p) ++r;
                while (r * (r + 1) / 2 > p) --r;
                const int i = p - r * (r + 1) / 2;
                if (i < r) A32[fsw(r, i)] = pa[s];
                T32[fsw(r, i)] = pm[s];  // M parked in the T region
            }
        }
        G::sync();
        if (warp >= 4 && warp < 8) {
            const int r0 = 16 * (warp & 3) + (lane >> 2);
#pragma unroll
            for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    accM[0][nt][e] = T32[fsw(r0 + (e >> 1) * 8, 8 * nt + 2 * (lane & 3) + (e & 1))];
        }
    }
    G::sync();

    wy_solve<NT, G>(A32, T32, reinterpret_cast<bf16 *>(T32));
    // M -> M16 (bf16, swizzled [64][64]; the second half of the T32 area)
    if (warp >= 4 && warp < 8) store_tile_bf16<8, 64>(accM, M16, 16 * (warp & 3), lane, 1.f);
    G::sync();
    return slow;
}

}  // namespace chunk
}  // namespace gdn2
