// The plain forward for few long sequences, split into sequence segments that
// run side by side.
//
// Per chunk the state update is affine in the state ("Why NVIDIA Gated
// DeltaNet-2 separates erase and write gates", section "Gated Delta Rule-2:
// per-channel erase/write split": S_t = (I - k (b . k)^T) Diag(alpha) S_{t-1}
// + k (w . v)^T), so over a segment of tokens S_end = Phi S_start + S_loc,
// where S_loc is the segment's end state from S_start = 0 and Phi (dk x dk) is
// its end state from S_start = I with the write term w . v set to zero; and
// for every token t in it, o_t = o_loc_t + S_start^T (Phi_t^T q_t), Phi_t the
// transition from the segment's start to t.  With B*H sequences too few to
// fill the GPU, each sequence is cut into P segments.
//
// dk = dv = 128 (the tensor-memory forward): segments are runs of whole
// chunks, as even as the chunk count allows, and
//   1. one launch runs the local pass of every segment (segment 0 from S0, so
//      its o and end state are final; the others from zero, o_loc written to
//      o) and the transition pass of segments 1..P-1 (start I, no write term;
//      Phi_t^T q_t per token and Phi), 2P - 1 CTAs per sequence side by side;
//   2. a scan in fp32 gives the start states S_start(p) = Phi(p-1) S_start(p-1)
//      + S_loc(p-1), S_start(1) = S_loc(0), and S_T = S_start(P);
//   3. a tensor-core pass adds S_start(p)^T (Phi_t^T q_t) to o in segments 1..P-1.
// About two forwards of work on 2P - 1 times as many SMs.
//
// Other head sizes (dk = dv = 64, the warp-level forward): P equal segments,
// S_loc and Phi from two forwards over the B*P segment-sequences (the
// transition pass reading a zero token tensor for v and w), the same scan,
// and a third forward for o and S_T from the true start states.
#include <algorithm>

#include "chunk_common.cuh"
#include "gdn2.h"
#include "launch.h"

namespace gdn2 {
namespace seg {

using chunk::bf16;

// Start states of the segments.  Block (b*H + h, column group g) owns 16
// value columns of one sequence and walks its P segments in order; each
// segment's transition is staged in shared memory (coalesced) before use.
constexpr int SCAN_COLS = 16, SCAN_THREADS = 256;
template <int DK>
__global__ void __launch_bounds__(SCAN_THREADS) scan_kernel(const float *S0, const float *Phi, const float *Sloc,
                                                           float *Sstart, int B, int H, int P, int dv) {
    extern __shared__ __align__(16) float sm[];
    // the transition with rows padded to DK + 1 floats: a warp's 32 rows fall in 32 banks
    float (*phi_s)[DK + 1] = reinterpret_cast<float (*)[DK + 1]>(sm);                         // [DK][DK + 1]
    float (*prev)[SCAN_COLS] = reinterpret_cast<float (*)[SCAN_COLS]>(sm + DK * (DK + 1));  // [DK][16]
    const int bh = blockIdx.x, b = bh / H, h = bh % H, c0 = blockIdx.y * SCAN_COLS;
    const int tid = threadIdx.x;
    constexpr int CPT = DK * SCAN_COLS / SCAN_THREADS;  // outputs per thread: CPT columns of one row
    const int r = tid % DK, cc = (tid / DK) * CPT;
    auto at = [&](int p) {  // offset of the [DK][dv] matrix of segment p of (b, h)
        return (((size_t)b * P + p) * H + h) * DK * dv;
    };
    for (int i = tid; i < DK * SCAN_COLS; i += SCAN_THREADS) {
        const int rr = i / SCAN_COLS, c = i % SCAN_COLS;
        const float v = S0 ? S0[(((size_t)b * H + h) * DK + rr) * dv + c0 + c] : 0.f;
        prev[rr][c] = v;
        Sstart[at(0) + (size_t)rr * dv + c0 + c] = v;
    }
    for (int p = 1; p < P; ++p) {
        const float4 *src = reinterpret_cast<const float4 *>(Phi + (((size_t)b * P + p - 1) * H + h) * DK * DK);
        for (int i = tid; i < DK * DK / 4; i += SCAN_THREADS) {
            const float4 t = src[i];
            const int rr = (4 * i) / DK, k = (4 * i) % DK;
            phi_s[rr][k] = t.x;
            phi_s[rr][k + 1] = t.y;
            phi_s[rr][k + 2] = t.z;
            phi_s[rr][k + 3] = t.w;
        }
        __syncthreads();  // the transition and prev are in place
        const float *loc = Sloc + at(p - 1) + (size_t)r * dv + c0 + cc;
        float acc[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) acc[j] = loc[j];
#pragma unroll 4
        for (int k = 0; k < DK; ++k) {
            const float a = phi_s[r][k];
#pragma unroll
            for (int j = 0; j < CPT; ++j) acc[j] += a * prev[k][cc + j];
        }
        __syncthreads();  // every thread is done reading the transition and prev
        float *out = Sstart + at(p) + (size_t)r * dv + c0 + cc;
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            prev[r][cc + j] = acc[j];
            out[j] = acc[j];
        }
    }
}

template <int DK>
constexpr int scan_smem_bytes() { return (DK * (DK + 1) + DK * SCAN_COLS) * (int)sizeof(float); }

// Start states of the segments of the tensor-memory path (one block per
// (b*H + h, column group)): S_start(1) = S_loc(0), S_start(p+1) = Phi(p)
// S_start(p) + S_loc(p); S_start(1..P-1) to Sstart[(b*(P-1) + p-1)*H + h] and
// S_start(P) = S_T.  The steps are sequential; each one's global loads (the
// next transition, the next S_loc columns) are issued into registers before
// the current step's product, so that their latency hides behind it.
template <int DK>
__global__ void __launch_bounds__(SCAN_THREADS) scan2_kernel(const float *Phi, const float *Sloc, float *Sstart,
                                                            float *S_T, int B, int H, int P, int dv) {
    extern __shared__ __align__(16) float sm[];
    float (*phi_s)[DK + 1] = reinterpret_cast<float (*)[DK + 1]>(sm);
    float (*prev)[SCAN_COLS] = reinterpret_cast<float (*)[SCAN_COLS]>(sm + DK * (DK + 1));
    const int bh = blockIdx.x, b = bh / H, h = bh % H, c0 = blockIdx.y * SCAN_COLS;
    const int tid = threadIdx.x;
    constexpr int CPT = DK * SCAN_COLS / SCAN_THREADS;
    constexpr int NPHI = DK * DK / 4 / SCAN_THREADS;  // float4 of a transition per thread
    const int r = tid % DK, cc = (tid / DK) * CPT;
    auto loc = [&](int p) { return Sloc + (((size_t)b * P + p) * H + h) * DK * dv; };
    auto phi = [&](int p) {
        return reinterpret_cast<const float4 *>(Phi + (((size_t)b * (P - 1) + p - 1) * H + h) * DK * DK);
    };
    float4 nphi[NPHI];  // the next transition
    float nloc[CPT];    // the next S_loc columns of this thread
    auto fetch = [&](int p) {  // (1 <= p < P)
        const float4 *src = phi(p);
#pragma unroll
        for (int j = 0; j < NPHI; ++j) nphi[j] = src[tid + j * SCAN_THREADS];
        const float *lp = loc(p) + (size_t)r * dv + c0 + cc;
#pragma unroll
        for (int j = 0; j < CPT; ++j) nloc[j] = lp[j];
    };
    if (P > 1) fetch(1);
    for (int i = tid; i < DK * SCAN_COLS; i += SCAN_THREADS) {
        const int rr = i / SCAN_COLS, c = i % SCAN_COLS;
        prev[rr][c] = loc(0)[(size_t)rr * dv + c0 + c];
    }
    for (int p = 1; p <= P; ++p) {
        __syncthreads();  // prev complete; every thread is done reading phi_s
        if (p < P) {
            float *out = Sstart + (((size_t)b * (P - 1) + p - 1) * H + h) * DK * dv;
            for (int i = tid; i < DK * SCAN_COLS; i += SCAN_THREADS)
                out[(size_t)(i / SCAN_COLS) * dv + c0 + i % SCAN_COLS] = prev[i / SCAN_COLS][i % SCAN_COLS];
        } else {
            if (S_T)
                for (int i = tid; i < DK * SCAN_COLS; i += SCAN_THREADS)
                    S_T[((size_t)b * H + h) * DK * dv + (size_t)(i / SCAN_COLS) * dv + c0 + i % SCAN_COLS] =
                        prev[i / SCAN_COLS][i % SCAN_COLS];
            break;
        }
#pragma unroll
        for (int j = 0; j < NPHI; ++j) {
            const int i4 = tid + j * SCAN_THREADS, rr = (4 * i4) / DK, k = (4 * i4) % DK;
            phi_s[rr][k] = nphi[j].x;
            phi_s[rr][k + 1] = nphi[j].y;
            phi_s[rr][k + 2] = nphi[j].z;
            phi_s[rr][k + 3] = nphi[j].w;
        }
        float acc[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) acc[j] = nloc[j];
        if (p + 1 < P) fetch(p + 1);  // in flight during this step's product
        __syncthreads();
#pragma unroll 4
        for (int k = 0; k < DK; ++k) {
            const float a = phi_s[r][k];
#pragma unroll
            for (int j = 0; j < CPT; ++j) acc[j] += a * prev[k][cc + j];
        }
        __syncthreads();  // every thread is done reading prev
#pragma unroll
        for (int j = 0; j < CPT; ++j) prev[r][cc + j] = acc[j];
    }
}

// o_t += S_start(p)^T (Phi_t^T q_t) for every token of segments 1..P-1: per
// block one (segment, head) and up to `tpb` 64-token tiles (chosen by the host
// so that the grid fills the SMs a few times over); the start state goes to
// shared memory once as bf16, each tile's rows Phi_t^T q_t arrive by cp.async
// one tile ahead, the product runs on the tensor cores (warp-level m16n8k16)
// into an fp32 tile in shared memory, and o is read (before the product, so
// that the load latency hides behind it), added to and written back with
// coalesced 16-byte accesses.  The pass is bound by the bytes of o and of
// those rows.
constexpr int kCorrMaxTiles = 16, kCorrThreads = 128;
constexpr int CORR_LD = 128 + 4;  // fp32 sum tile row pitch (rows 4 banks apart)
constexpr int CORR_SMEM = 128 * 128 * 2 + 2 * 64 * 128 * 2 + 64 * CORR_LD * 4;
__global__ void __launch_bounds__(kCorrThreads) correct_kernel(const bf16 *qphi, const float *Sstart, bf16 *o, int B,
                                                               int T, int H, int P, int tpb) {
    constexpr int D = 128;
    extern __shared__ __align__(1024) unsigned char smc[];
    bf16 *S16 = reinterpret_cast<bf16 *>(smc);                                  // [128 k][128 n], swizzled
    auto Qb = [&](int par) {  // [64 t][128 k], swizzled, by tile parity
        return reinterpret_cast<bf16 *>(smc + D * D * 2 + par * (64 * D * 2));
    };
    float *acc_s = reinterpret_cast<float *>(smc + D * D * 2 + 2 * 64 * D * 2);  // [64 t][CORR_LD] fp32
    const int seg = blockIdx.y / H, h = blockIdx.y % H;                    // seg = b*(P-1) + p - 1
    const int b = seg / (P - 1), p = seg % (P - 1) + 1;
    const int nch = T / chunk::C, base = nch / P, rem = nch % P;
    const int c0 = p * base + min(p, rem), cn = base + (p < rem ? 1 : 0);
    const int t0 = blockIdx.x * tpb;
    if (t0 >= cn) return;
    const int ntl = min(cn, t0 + tpb) - t0;
    const size_t row0 = (size_t)b * T + (size_t)c0 * chunk::C;
    const float4 *Ss = reinterpret_cast<const float4 *>(Sstart + ((size_t)seg * H + h) * D * D);
    for (int i = threadIdx.x; i < D * D / 4; i += kCorrThreads) {
        const float4 v = Ss[i];
        const int k = (4 * i) / D, n = (4 * i) % D;
        *reinterpret_cast<uint2 *>(S16 + chunk::swz<D, D>(k, n)) =
            make_uint2(chunk::pack_bf16(v.x, v.y), chunk::pack_bf16(v.z, v.w));
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int IT = 64 * D / 8 / kCorrThreads;
    chunk::load_token_tile<D, kCorrThreads>(Qb(0), qphi, row0, cn * chunk::C, h, t0, H);
    chunk::cp_commit();
    for (int i = 0; i < ntl; ++i) {
        const int tl = t0 + i;
        // the next tile's rows into the other buffer (its last reader, the
        // product two tiles back, is behind the barrier that ended that tile)
        if (i + 1 < ntl) chunk::load_token_tile<D, kCorrThreads>(Qb((i + 1) & 1), qphi, row0, cn * chunk::C, h, tl + 1, H);
        chunk::cp_commit();
        // this tile's o rows (16 bytes per access), in flight during the product
        uint4 ov[IT];
        uint4 *op[IT];
#pragma unroll
        for (int it = 0; it < IT; ++it) {
            const int id = threadIdx.x + it * kCorrThreads, rr = id / (D / 8), cc = (id % (D / 8)) * 8;
            op[it] = reinterpret_cast<uint4 *>(o + ((row0 + (size_t)tl * chunk::C + rr) * H + h) * D + cc);
            ov[it] = *op[it];
        }
        chunk::cp_wait<1>();  // this tile's rows (the group before the one just committed)
        __syncthreads();      // (and S16; the previous tile's sums read)
        float acc[1][16][4];
        chunk::zero(acc);
        chunk::warp_gemm<1, 16, true, false, D, D, 64, D>(acc, Qb(i & 1), 16 * warp, S16, 0, D, lane);
        const int r = 16 * warp + (lane >> 2);
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            const int c = 8 * nt + 2 * (lane & 3);
            *reinterpret_cast<float2 *>(acc_s + r * CORR_LD + c) = make_float2(acc[0][nt][0], acc[0][nt][1]);
            *reinterpret_cast<float2 *>(acc_s + (r + 8) * CORR_LD + c) = make_float2(acc[0][nt][2], acc[0][nt][3]);
        }
        __syncthreads();
#pragma unroll
        for (int it = 0; it < IT; ++it) {
            const int id = threadIdx.x + it * kCorrThreads, rr = id / (D / 8), cc = (id % (D / 8)) * 8;
            const float4 a0 = *reinterpret_cast<const float4 *>(acc_s + rr * CORR_LD + cc);
            const float4 a1 = *reinterpret_cast<const float4 *>(acc_s + rr * CORR_LD + cc + 4);
            const float2 x0 = chunk::unpack_bf16(ov[it].x), x1 = chunk::unpack_bf16(ov[it].y);
            const float2 x2 = chunk::unpack_bf16(ov[it].z), x3 = chunk::unpack_bf16(ov[it].w);
            *op[it] = make_uint4(chunk::pack_bf16(x0.x + a0.x, x0.y + a0.y), chunk::pack_bf16(x1.x + a0.z, x1.y + a0.w),
                                 chunk::pack_bf16(x2.x + a1.x, x2.y + a1.y), chunk::pack_bf16(x3.x + a1.z, x3.y + a1.w));
        }
    }
}

// ---- segmented training (the saved-state pair, dk = dv = 128)

// Offsets of the B*P segments as a packed batch over the B*T token rows.
__global__ void seg_cu_kernel(int *cu, int B, int T, int P) {
    const int nch = T / chunk::C, base = nch / P, rem = nch % P;
    for (int n = blockIdx.x * blockDim.x + threadIdx.x; n <= B * P; n += gridDim.x * blockDim.x) {
        if (n == B * P) {
            cu[n] = B * T;
        } else {
            const int b = n / P, p = n % P;
            cu[n] = b * T + chunk::C * (p * base + min(p, rem));
        }
    }
}

// The start states of the segments, per (b*P + p, head h): p == 0 from S0
// (a [B][H] array, nullptr = zero), p >= 1 from `later` (a [B*(P-1)][H] array).
__global__ void seg_gather_kernel(const float *first, const float *later, float *out, int B, int H, int P) {
    constexpr int DD = 128 * 128;
    const size_t n = (size_t)B * P * H * DD;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const size_t m = i / DD, e = i % DD;
        const int h = (int)(m % H), bp = (int)(m / H), b = bp / P, p = bp % P;
        float v = 0.f;
        if (p == 0) {
            if (first) v = first[((size_t)b * H + h) * DD + e];
        } else if (later) {
            v = later[(((size_t)b * (P - 1) + p - 1) * H + h) * DD + e];
        }
        out[i] = v;
    }
}

// dS0 [B][H] = the first segment's start-state gradient of each sequence.
__global__ void seg_first_kernel(const float *seg, float *out, int B, int H, int P) {
    constexpr int DD = 128 * 128;
    const size_t n = (size_t)B * H * DD;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const size_t m = i / DD, e = i % DD;
        const int b = (int)(m / H), h = (int)(m % H);
        out[i] = seg[(((size_t)b * P) * H + h) * DD + e];
    }
}

// End-state gradients of the segments, last to first: G(P-1) = dS_T,
// G(p) = Phi(p+1)^T G(p+1) + L(p+1), with L(q) the start-state gradient of
// segment q from a zero end gradient.  One block per (b*H + h, column
// group), as the forward scan.
template <int DK>
__global__ void __launch_bounds__(SCAN_THREADS) rscan_kernel(const float *Phi, const float *L, const float *dS_T,
                                                            float *G, int B, int H, int P) {
    extern __shared__ __align__(16) float sm[];
    float (*phit)[DK + 1] = reinterpret_cast<float (*)[DK + 1]>(sm);  // Phi^T, padded rows
    float (*prev)[SCAN_COLS] = reinterpret_cast<float (*)[SCAN_COLS]>(sm + DK * (DK + 1));
    const int bh = blockIdx.x, b = bh / H, h = bh % H, c0 = blockIdx.y * SCAN_COLS;
    const int tid = threadIdx.x;
    constexpr int CPT = DK * SCAN_COLS / SCAN_THREADS;
    const int r = tid % DK, cc = (tid / DK) * CPT;
    auto at = [&](int p) { return (((size_t)b * P + p) * H + h) * DK * DK; };
    for (int i = tid; i < DK * SCAN_COLS; i += SCAN_THREADS) {
        const int rr = i / SCAN_COLS, c = i % SCAN_COLS;
        prev[rr][c] = dS_T ? dS_T[((size_t)b * H + h) * DK * DK + (size_t)rr * DK + c0 + c] : 0.f;
    }
    for (int p = P - 1; p >= 0; --p) {
        __syncthreads();  // prev complete
        for (int i = tid; i < DK * SCAN_COLS; i += SCAN_THREADS)
            G[at(p) + (size_t)(i / SCAN_COLS) * DK + c0 + i % SCAN_COLS] = prev[i / SCAN_COLS][i % SCAN_COLS];
        if (p == 0) break;
        // Phi(p) (stored at (b*(P-1) + p-1)*H + h) transposed into shared memory
        const float4 *src = reinterpret_cast<const float4 *>(Phi + (((size_t)b * (P - 1) + p - 1) * H + h) * DK * DK);
        for (int i = tid; i < DK * DK / 4; i += SCAN_THREADS) {
            const float4 t = src[i];
            const int rr = (4 * i) / DK, k = (4 * i) % DK;
            phit[k][rr] = t.x;
            phit[k + 1][rr] = t.y;
            phit[k + 2][rr] = t.z;
            phit[k + 3][rr] = t.w;
        }
        __syncthreads();
        const float *lp = L + at(p) + (size_t)r * DK + c0 + cc;
        float acc[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) acc[j] = lp[j];
#pragma unroll 4
        for (int k = 0; k < DK; ++k) {
            const float a = phit[r][k];
#pragma unroll
            for (int j = 0; j < CPT; ++j) acc[j] += a * prev[k][cc + j];
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < CPT; ++j) prev[r][cc + j] = acc[j];
    }
}

struct Carve {
    float *fwd_ws;
    float *phi, *sloc, *sstart;
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Byte layout of the segmented path's workspace (p == nullptr: sizes only).
size_t carve(void *p, int B, int T, int H, int dk, int dv, int P, Carve *c) {
    const size_t Bp = (size_t)B * P;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += align256(bytes);
        return p ? static_cast<unsigned char *>(p) + at : nullptr;
    };
    unsigned char *fw = take(chunk_fwd_ws_bytes((int)Bp, H, dk));
    unsigned char *ph = take(Bp * H * dk * dk * sizeof(float));
    unsigned char *sl = take(Bp * H * dk * dv * sizeof(float));
    unsigned char *ss = take(Bp * H * dk * dv * sizeof(float));
    if (c) *c = {reinterpret_cast<float *>(fw), reinterpret_cast<float *>(ph), reinterpret_cast<float *>(sl),
                 reinterpret_cast<float *>(ss)};
    return off;
}

// ... and of the tensor-memory path (dk = dv = 128): the forward's per-CTA
// scratch for B*H*(2P - 1) CTAs, the rows Phi_t^T q_t (bf16, laid out like
// o), S_loc of every segment, Phi and S_start of segments 1..P-1.
struct Carve2 {
    float *fwd_ws;
    bf16 *qphi;
    float *sloc, *phi, *sstart;
};
size_t carve2(void *p, int B, int T, int H, int P, Carve2 *c) {
    constexpr int D = 128;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += align256(bytes);
        return p ? static_cast<unsigned char *>(p) + at : nullptr;
    };
    unsigned char *fw = take(chunk_fwd_ws_bytes(B * (2 * P - 1), H, D));
    unsigned char *q = take((size_t)B * T * H * D * sizeof(bf16));
    unsigned char *sl = take((size_t)B * P * H * D * D * sizeof(float));
    unsigned char *ph = take((size_t)B * (P - 1) * H * D * D * sizeof(float));
    unsigned char *ss = take((size_t)B * (P - 1) * H * D * D * sizeof(float));
    if (c) *c = {reinterpret_cast<float *>(fw), reinterpret_cast<bf16 *>(q), reinterpret_cast<float *>(sl),
                 reinterpret_cast<float *>(ph), reinterpret_cast<float *>(ss)};
    return off;
}

int num_sms() {
    static int n = [] {
        int dev = 0, v = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) !=
                                                      cudaSuccess) {
            (void)cudaGetLastError();
            return 148;
        }
        return v;
    }();
    return n;
}

}  // namespace seg

int segment_count(int B, int T, int H, int dk, int dv) {
    if (dk != dv || B <= 0 || H <= 0 || T <= 0) return 1;
    const long long seqs = (long long)B * H, sms = seg::num_sms();
    if (dk == 128) {
        // local and transition passes side by side: B*H*(2P - 1) CTAs in one
        // wave, segments of at least 8 whole chunks
        if (T % chunk::C) return 1;
        int P = 1;
        while (seqs * (2 * (P + 1) - 1) <= sms && T / chunk::C >= 8 * (P + 1)) ++P;
        return P;
    }
    int P = 1;
    // double while the segment-sequences still fit in one wave and every
    // segment keeps at least 8 whole chunks
    while (seqs * P * 2 <= sms && T % (2 * P * chunk::C) == 0 && T / (2 * P) >= 8 * chunk::C) P *= 2;
    return P >= 4 ? P : 1;  // the three passes pay off from four segments on
}

size_t segments_ws_bytes(int B, int T, int H, int dk, int dv, int P) {
    if (dk == 128 && dv == 128) return seg::carve2(nullptr, B, T, H, P, nullptr);
    return seg::carve(nullptr, B, T, H, dk, dv, P, nullptr);
}

cudaError_t launch_chunk_fwd_segments(const ChunkFwdArgs &a, int dk, int dv, int P, void *ws, cudaStream_t s) {
    cudaError_t e;
    if (dk == 128 && dv == 128) {
        seg::Carve2 c;
        seg::carve2(ws, a.B, a.T, a.H, P, &c);
        // 1. local passes of every segment and transition passes of segments 1..P-1, one launch
        ChunkFwdArgs f = a;
        f.ws = c.fwd_ws;
        f.ws_stride = (size_t)chunk::C * 128;
        f.S_T = nullptr;
        f.seg_P = P;
        f.seg_loc = c.sloc;
        f.seg_phi = c.phi;
        f.seg_qphi = c.qphi;
        if ((e = launch_chunk_fwd_tc(f, s)) != cudaSuccess) return e;
        // 2. start states of segments 1..P-1 and S_T
        constexpr int bytes = seg::scan_smem_bytes<128>();
        if ((e = cudaFuncSetAttribute(seg::scan2_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) !=
            cudaSuccess)
            return e;
        seg::scan2_kernel<128><<<dim3((unsigned)(a.B * a.H), 128 / seg::SCAN_COLS), seg::SCAN_THREADS, bytes, s>>>(
            c.phi, c.sloc, c.sstart, a.S_T, a.B, a.H, P, 128);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        // 3. o += S_start^T (Phi_t^T q_t) in segments 1..P-1
        if (a.o) {
            const int longest = (a.T / chunk::C + P - 1) / P;  // chunks of the longest segment
            if ((e = cudaFuncSetAttribute(seg::correct_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          seg::CORR_SMEM)) != cudaSuccess)
                return e;
            // tiles per block: about four blocks per SM (two resident at a time)
            const long long tiles = (long long)longest * a.B * (P - 1) * a.H;
            const int tpb = (int)std::max(1LL, std::min<long long>(seg::kCorrMaxTiles,
                                                                  (tiles + 4LL * seg::num_sms() - 1) / (4LL * seg::num_sms())));
            seg::correct_kernel<<<dim3((unsigned)((longest + tpb - 1) / tpb), (unsigned)(a.B * (P - 1) * a.H)),
                                  seg::kCorrThreads, seg::CORR_SMEM, s>>>(
                c.qphi, c.sstart, static_cast<seg::bf16 *>(a.o), a.B, a.T, a.H, P, tpb);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    seg::Carve c;
    seg::carve(ws, a.B, a.T, a.H, dk, dv, P, &c);
    const int Bp = a.B * P, Tp = a.T / P;
    const size_t wstride = (size_t)chunk::C * dk;
    // 1. every segment from a zero start (S_loc) and its transition (Phi: start I,
    // no write term; the kernel reads no v and w for it)
    ChunkFwdArgs loc{a.q, a.k, a.v, a.log_alpha, a.b, a.w, nullptr, nullptr, c.sloc, c.fwd_ws, wstride,
                     nullptr, nullptr, nullptr, a.status, Bp, Tp, a.H};
    if ((e = launch_chunk_fwd(loc, dk, dv, s)) != cudaSuccess) return e;
    ChunkFwdArgs phi{a.q, a.k, a.v, a.log_alpha, a.b, a.w, nullptr, nullptr, c.phi, c.fwd_ws, wstride,
                     nullptr, nullptr, nullptr, a.status, Bp, Tp, a.H};
    phi.transition = true;
    if ((e = launch_chunk_fwd(phi, dk, dk, s)) != cudaSuccess) return e;
    // 2. the segments' start states
    const dim3 grid((unsigned)(a.B * a.H), (unsigned)(dv / seg::SCAN_COLS));
    if (dk == 128) {
        constexpr int bytes = seg::scan_smem_bytes<128>();
        if ((e = cudaFuncSetAttribute(seg::scan_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) !=
            cudaSuccess)
            return e;
        seg::scan_kernel<128><<<grid, seg::SCAN_THREADS, bytes, s>>>(a.S0, c.phi, c.sloc, c.sstart, a.B, a.H, P, dv);
    } else {
        constexpr int bytes = seg::scan_smem_bytes<64>();
        seg::scan_kernel<64><<<grid, seg::SCAN_THREADS, bytes, s>>>(a.S0, c.phi, c.sloc, c.sstart, a.B, a.H, P, dv);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 3. o and the segments' end states from the true start states
    ChunkFwdArgs fin{a.q, a.k, a.v, a.log_alpha, a.b, a.w, c.sstart, a.o, c.sloc, c.fwd_ws, wstride,
                     nullptr, nullptr, nullptr, a.status, Bp, Tp, a.H};
    if ((e = launch_chunk_fwd(fin, dk, dv, s)) != cudaSuccess) return e;
    // S_T = the end state of every sequence's last segment (one copy per batch)
    if (a.S_T) {
        const size_t per = (size_t)a.H * dk * dv;
        for (int b = 0; b < a.B; ++b) {
            e = cudaMemcpyAsync(a.S_T + (size_t)b * per, c.sloc + ((size_t)b * P + P - 1) * per, per * sizeof(float),
                                cudaMemcpyDeviceToDevice, s);
            if (e != cudaSuccess) return e;
        }
    }
    return cudaSuccess;
}

// ---------------------------------------------------------------------------
// Segmented training: the saved-state pair for few long sequences (dk = dv =
// 128, bf16).  The forward finds every segment's start state with the
// segment path (local and transition passes, the scan), then runs the saving
// forward over the B*P segments as a packed batch from those start states.
// The backward runs the packed backward twice: first with zero end gradients
// (each segment's own start-state gradient L), then, after a reverse scan
// G(p) = Phi(p+1)^T G(p+1) + L(p+1), with the true end gradients G.

namespace seg {

struct TrainFwdCarve {
    Carve2 c2;
    float *s0seg;
    int *cu;
    float *fwd_ws;
};
size_t carve_train_fwd(void *p, int B, int T, int H, int P, TrainFwdCarve *c) {
    constexpr int D = 128;
    Carve2 c2{};
    size_t off = align256(carve2(p, B, T, H, P, &c2));
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += align256(bytes);
        return p ? static_cast<unsigned char *>(p) + at : nullptr;
    };
    unsigned char *s0 = take((size_t)B * P * H * D * D * sizeof(float));
    unsigned char *cu = take(((size_t)B * P + 1) * sizeof(int));
    unsigned char *fw = take(chunk_fwd_ws_bytes(B * P, H, D));
    if (c) *c = {c2, reinterpret_cast<float *>(s0), reinterpret_cast<int *>(cu), reinterpret_cast<float *>(fw)};
    return off;
}

struct TrainBwdCarve {
    float *scratch;
    size_t stride;
    float *dst_seg, *l_seg, *g_seg;
    int *cu;
};
size_t carve_train_bwd(void *p, int B, int T, int H, int P, TrainBwdCarve *c) {
    constexpr int D = 128;
    size_t stride = 0, sbytes = 0;
    const size_t scr = chunk_bwd_ws_bytes(B * P, B * T, H, D, D, &stride, &sbytes, true) - sbytes;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += align256(bytes);
        return p ? static_cast<unsigned char *>(p) + at : nullptr;
    };
    unsigned char *sc = take(scr);
    unsigned char *d = take((size_t)B * P * H * D * D * sizeof(float));
    unsigned char *l = take((size_t)B * P * H * D * D * sizeof(float));
    unsigned char *g = take((size_t)B * P * H * D * D * sizeof(float));
    unsigned char *cu = take(((size_t)B * P + 1) * sizeof(int));
    if (c)
        *c = {reinterpret_cast<float *>(sc), stride, reinterpret_cast<float *>(d), reinterpret_cast<float *>(l),
              reinterpret_cast<float *>(g), reinterpret_cast<int *>(cu)};
    return off;
}

unsigned grid_for(size_t n) { return (unsigned)std::min<size_t>((n + 255) / 256, 4096); }

}  // namespace seg

int seg_train_count(int B, int T, int H, int dk, int dv) {
    return (dk == 128 && dv == 128) ? segment_count(B, T, H, dk, dv) : 1;
}

// The saved buffer of segmented training: the packed batch's states, tiles
// and decayed operands (the layout of the _varlen pair for B*P sequences
// over B*T rows), then the transitions Phi of segments 1..P-1.
size_t seg_train_states_bytes(int B, int T, int H, int P) {
    const int N = B * P, R = B * T;
    return states_region_bytes(N, R, H, 128, 128, true) + intra_region_bytes(N, R, H, 128, true) +
           (ops_region_bytes(N, R, H, 128, 128, true) + 255) / 256 * 256 +
           (size_t)B * (P - 1) * H * 128 * 128 * sizeof(float);
}
size_t seg_train_fwd_ws_bytes(int B, int T, int H, int P) { return seg::carve_train_fwd(nullptr, B, T, H, P, nullptr); }
size_t seg_train_bwd_ws_bytes(int B, int T, int H, int P) { return seg::carve_train_bwd(nullptr, B, T, H, P, nullptr); }

namespace {
// the regions of the segmented-training saved buffer
void train_regions(void *states, int B, int T, int H, int P, char **st, char **intra, char **ops, float **phi) {
    const int N = B * P, R = B * T;
    char *base = static_cast<char *>(states);
    *st = base;
    *intra = base + states_region_bytes(N, R, H, 128, 128, true);
    *ops = *intra + intra_region_bytes(N, R, H, 128, true);
    *phi = reinterpret_cast<float *>(*ops + (ops_region_bytes(N, R, H, 128, 128, true) + 255) / 256 * 256);
}
}  // namespace

cudaError_t launch_seg_train_fwd(const ChunkFwdArgs &a, void *states, int P, void *ws, cudaStream_t s) {
    constexpr int D = 128;
    seg::TrainFwdCarve c;
    seg::carve_train_fwd(ws, a.B, a.T, a.H, P, &c);
    char *st, *intra, *ops;
    float *phi;
    train_regions(states, a.B, a.T, a.H, P, &st, &intra, &ops, &phi);
    cudaError_t e;
    // 1. every segment's local pass and the transitions (into the saved buffer), then the scan
    ChunkFwdArgs f = a;
    f.ws = c.c2.fwd_ws;
    f.ws_stride = (size_t)chunk::C * D;
    f.S_T = nullptr;
    f.states = f.intra = f.ops = nullptr;
    f.seg_P = P;
    f.seg_loc = c.c2.sloc;
    f.seg_phi = phi;
    f.seg_qphi = c.c2.qphi;
    if ((e = launch_chunk_fwd_tc(f, s)) != cudaSuccess) return e;
    constexpr int bytes = seg::scan_smem_bytes<D>();
    if ((e = cudaFuncSetAttribute(seg::scan2_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) !=
        cudaSuccess)
        return e;
    seg::scan2_kernel<D><<<dim3((unsigned)(a.B * a.H), D / seg::SCAN_COLS), seg::SCAN_THREADS, bytes, s>>>(
        phi, c.c2.sloc, c.c2.sstart, a.S_T, a.B, a.H, P, D);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 2. the segments as a packed batch from their start states, keeping what the backward needs
    const size_t nseg = (size_t)a.B * P * a.H * D * D;
    seg::seg_gather_kernel<<<seg::grid_for(nseg), 256, 0, s>>>(a.S0, c.c2.sstart, c.s0seg, a.B, a.H, P);
    seg::seg_cu_kernel<<<1, 256, 0, s>>>(c.cu, a.B, a.T, P);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    ChunkFwdArgs g{a.q, a.k, a.v, a.log_alpha, a.b, a.w, c.s0seg, a.o, nullptr, c.fwd_ws, (size_t)chunk::C * D,
                   st, intra, ops, a.status, a.B * P, a.B * a.T, a.H, c.cu};
    g.wait_limit = a.wait_limit;
    return launch_chunk_fwd_tc(g, s);
}

cudaError_t launch_seg_train_bwd(const ChunkBwdArgs &a, const void *states, int P, void *ws, cudaStream_t s) {
    constexpr int D = 128;
    seg::TrainBwdCarve c;
    seg::carve_train_bwd(ws, a.B, a.T, a.H, P, &c);
    char *st, *intra, *ops;
    float *phi;
    train_regions(const_cast<void *>(states), a.B, a.T, a.H, P, &st, &intra, &ops, &phi);
    cudaError_t e;
    const size_t nseg = (size_t)a.B * P * a.H * D * D;
    seg::seg_cu_kernel<<<1, 256, 0, s>>>(c.cu, a.B, a.T, P);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(c.dst_seg, 0, nseg * sizeof(float), s)) != cudaSuccess) return e;
    ChunkBwdArgs b{a.q, a.k, a.v, a.log_alpha, a.b, a.w, nullptr, a.dO, c.dst_seg, a.dq, a.dk, a.dv, a.dlog_alpha,
                   a.db, a.dw, c.l_seg, st, intra, ops, c.scratch, c.stride, a.status, 1, a.B * P, a.B * a.T, a.H,
                   c.cu};
    b.wait_limit = a.wait_limit;
    // 1. every segment from a zero end gradient: its own start-state gradient L
    if ((e = launch_chunk_bwd_tc(b, s)) != cudaSuccess) return e;
    // 2. the true end gradients, last segment to first
    constexpr int bytes = seg::scan_smem_bytes<D>();
    if ((e = cudaFuncSetAttribute(seg::rscan_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) !=
        cudaSuccess)
        return e;
    seg::rscan_kernel<D><<<dim3((unsigned)(a.B * a.H), D / seg::SCAN_COLS), seg::SCAN_THREADS, bytes, s>>>(
        phi, c.l_seg, a.dS_T, c.g_seg, a.B, a.H, P);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 3. every segment again from its true end gradient: the gradients, and dS0 of the first
    b.dS_T = c.g_seg;
    b.dS0 = c.l_seg;
    if ((e = launch_chunk_bwd_tc(b, s)) != cudaSuccess) return e;
    if (a.dS0) {
        seg::seg_first_kernel<<<seg::grid_for((size_t)a.B * a.H * D * D), 256, 0, s>>>(c.l_seg, a.dS0, a.B, a.H, P);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace gdn2
