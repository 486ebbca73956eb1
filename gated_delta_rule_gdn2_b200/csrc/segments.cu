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

// Identity matrices [count][d][d] (fp32).
__global__ void identity_kernel(float *m, size_t count, int d) {
    const size_t n = count * d * d;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const size_t e = i % ((size_t)d * d);
        m[i] = (e / d == e % d) ? 1.f : 0.f;
    }
}

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
// S_start(P) = S_T.
template <int DK>
__global__ void __launch_bounds__(SCAN_THREADS) scan2_kernel(const float *Phi, const float *Sloc, float *Sstart,
                                                            float *S_T, int B, int H, int P, int dv) {
    extern __shared__ __align__(16) float sm[];
    float (*phi_s)[DK + 1] = reinterpret_cast<float (*)[DK + 1]>(sm);
    float (*prev)[SCAN_COLS] = reinterpret_cast<float (*)[SCAN_COLS]>(sm + DK * (DK + 1));
    const int bh = blockIdx.x, b = bh / H, h = bh % H, c0 = blockIdx.y * SCAN_COLS;
    const int tid = threadIdx.x;
    constexpr int CPT = DK * SCAN_COLS / SCAN_THREADS;
    const int r = tid % DK, cc = (tid / DK) * CPT;
    auto loc = [&](int p) { return Sloc + (((size_t)b * P + p) * H + h) * DK * dv; };
    for (int i = tid; i < DK * SCAN_COLS; i += SCAN_THREADS) {
        const int rr = i / SCAN_COLS, c = i % SCAN_COLS;
        prev[rr][c] = loc(0)[(size_t)rr * dv + c0 + c];
    }
    for (int p = 1; p <= P; ++p) {
        __syncthreads();  // prev complete
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
        const float4 *src = reinterpret_cast<const float4 *>(Phi + (((size_t)b * (P - 1) + p - 1) * H + h) * DK * DK);
        for (int i = tid; i < DK * DK / 4; i += SCAN_THREADS) {
            const float4 t = src[i];
            const int rr = (4 * i) / DK, k = (4 * i) % DK;
            phi_s[rr][k] = t.x;
            phi_s[rr][k + 1] = t.y;
            phi_s[rr][k + 2] = t.z;
            phi_s[rr][k + 3] = t.w;
        }
        __syncthreads();
        const float *lp = loc(p) + (size_t)r * dv + c0 + cc;
        float acc[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) acc[j] = lp[j];
#pragma unroll 4
        for (int k = 0; k < DK; ++k) {
            const float a = phi_s[r][k];
#pragma unroll
            for (int j = 0; j < CPT; ++j) acc[j] += a * prev[k][cc + j];
        }
        __syncthreads();  // every thread is done reading Phi and prev
#pragma unroll
        for (int j = 0; j < CPT; ++j) prev[r][cc + j] = acc[j];
    }
}

// o_t += S_start(p)^T (Phi_t^T q_t) for every token of segments 1..P-1: per
// block one (segment, head) and up to kCorrTiles 64-token tiles; the start
// state goes to shared memory once as bf16, each tile's rows Phi_t^T q_t
// arrive by cp.async, and the product runs on the tensor cores (warp-level
// m16n8k16; the pass is bound by the bytes of o and of those rows).
constexpr int kCorrTiles = 8, kCorrThreads = 128;
constexpr int CORR_SMEM = 128 * 128 * 2 + 64 * 128 * 2;
__global__ void __launch_bounds__(kCorrThreads) correct_kernel(const bf16 *qphi, const float *Sstart, bf16 *o, int B,
                                                               int T, int H, int P) {
    constexpr int D = 128;
    extern __shared__ __align__(1024) unsigned char smc[];
    bf16 *S16 = reinterpret_cast<bf16 *>(smc);              // [128 k][128 n], swizzled
    bf16 *Q16 = reinterpret_cast<bf16 *>(smc + D * D * 2);   // [64 t][128 k], swizzled
    const int seg = blockIdx.y / H, h = blockIdx.y % H;      // seg = b*(P-1) + p - 1
    const int b = seg / (P - 1), p = seg % (P - 1) + 1;
    const int nch = T / chunk::C, base = nch / P, rem = nch % P;
    const int c0 = p * base + min(p, rem), cn = base + (p < rem ? 1 : 0);
    const int t0 = blockIdx.x * kCorrTiles;
    if (t0 >= cn) return;
    const size_t row0 = (size_t)b * T + (size_t)c0 * chunk::C;
    const float *Ss = Sstart + ((size_t)seg * H + h) * D * D;
    for (int i = threadIdx.x; i < D * D / 2; i += kCorrThreads) {
        const int k = (2 * i) / D, n = (2 * i) % D;
        const float2 v = *reinterpret_cast<const float2 *>(Ss + (size_t)k * D + n);
        *reinterpret_cast<uint32_t *>(S16 + chunk::swz<D, D>(k, n)) = chunk::pack_bf16(v.x, v.y);
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int tl = t0; tl < min(cn, t0 + kCorrTiles); ++tl) {
        __syncthreads();  // (S16 written; the previous tile's rows read)
        chunk::load_token_tile<D, kCorrThreads>(Q16, qphi, row0, cn * chunk::C, h, tl, H);
        chunk::cp_commit();
        chunk::cp_wait<0>();
        __syncthreads();
        float acc[1][16][4];
        chunk::zero(acc);
        chunk::warp_gemm<1, 16, true, false, D, D, 64, D>(acc, Q16, 16 * warp, S16, 0, D, lane);
        const int r = 16 * warp + (lane >> 2);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            bf16 *orow = o + ((row0 + (size_t)tl * chunk::C + r + 8 * half) * H + h) * D;
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                const int c = 8 * nt + 2 * (lane & 3);
                __nv_bfloat162 *pr = reinterpret_cast<__nv_bfloat162 *>(orow + c);
                const float2 ov = __bfloat1622float2(*pr);
                *pr = __floats2bfloat162_rn(ov.x + acc[0][nt][2 * half], ov.y + acc[0][nt][2 * half + 1]);
            }
        }
    }
}

struct Carve {
    float *fwd_ws;
    bf16 *zeros;
    float *ident, *phi, *sloc, *sstart;
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
    unsigned char *z = take((size_t)B * T * H * dk * sizeof(bf16));
    unsigned char *id = take(Bp * H * dk * dk * sizeof(float));
    unsigned char *ph = take(Bp * H * dk * dk * sizeof(float));
    unsigned char *sl = take(Bp * H * dk * dv * sizeof(float));
    unsigned char *ss = take(Bp * H * dk * dv * sizeof(float));
    if (c) *c = {reinterpret_cast<float *>(fw), reinterpret_cast<bf16 *>(z), reinterpret_cast<float *>(id),
                 reinterpret_cast<float *>(ph), reinterpret_cast<float *>(sl), reinterpret_cast<float *>(ss)};
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
            seg::correct_kernel<<<dim3((unsigned)((longest + seg::kCorrTiles - 1) / seg::kCorrTiles),
                                       (unsigned)(a.B * (P - 1) * a.H)),
                                  seg::kCorrThreads, seg::CORR_SMEM, s>>>(
                c.qphi, c.sstart, static_cast<seg::bf16 *>(a.o), a.B, a.T, a.H, P);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    seg::Carve c;
    seg::carve(ws, a.B, a.T, a.H, dk, dv, P, &c);
    const int Bp = a.B * P, Tp = a.T / P;
    const size_t wstride = (size_t)chunk::C * dk;
    e = cudaMemsetAsync(c.zeros, 0, (size_t)a.B * a.T * a.H * dk * sizeof(seg::bf16), s);
    if (e != cudaSuccess) return e;
    const size_t nident = (size_t)Bp * a.H;
    seg::identity_kernel<<<(unsigned)std::min<size_t>((nident * dk * dk + 255) / 256, 4096), 256, 0, s>>>(
        c.ident, nident, dk);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 1. every segment from a zero start (S_loc) and its transition (Phi: start I, no write term)
    ChunkFwdArgs loc{a.q, a.k, a.v, a.log_alpha, a.b, a.w, nullptr, nullptr, c.sloc, c.fwd_ws, wstride,
                     nullptr, nullptr, nullptr, a.status, Bp, Tp, a.H};
    if ((e = launch_chunk_fwd(loc, dk, dv, s)) != cudaSuccess) return e;
    ChunkFwdArgs phi{a.q, a.k, c.zeros, a.log_alpha, a.b, c.zeros, c.ident, nullptr, c.phi, c.fwd_ws, wstride,
                     nullptr, nullptr, nullptr, a.status, Bp, Tp, a.H};
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

}  // namespace gdn2
