// The plain forward for few long sequences, split into sequence segments that
// run side by side.
//
// Per chunk the state update is affine in the state ("Why NVIDIA Gated
// DeltaNet-2 separates erase and write gates", section "Gated Delta Rule-2:
// per-channel erase/write split": S_t = (I - k (b . k)^T) Diag(alpha) S_{t-1}
// + k (w . v)^T), so over a segment of tokens S_end = Phi S_start + S_loc,
// where S_loc is the segment's end state from S_start = 0 and Phi (dk x dk) is
// its end state from S_start = I with the write term w . v set to zero.  With
// B*H sequences too few to fill the GPU, each sequence is cut into P equal
// segments and
//   1. S_loc and Phi of every segment come from two forwards over the B*P
//      segment-sequences (a segment of batch b is batch b*P + p of the same
//      [B, T, H, D] buffers read as [B*P, T/P, H, D]);
//   2. a scan in fp32 gives every segment's start state,
//      S_start(p) = Phi(p-1) S_start(p-1) + S_loc(p-1), S_start(0) = S0;
//   3. a third forward from those start states gives o and the end states.
// The work is about three forwards, spread over P times as many CTAs.
#include <algorithm>

#include "chunk_common.cuh"
#include "gdn2.h"
#include "launch.h"

namespace gdn2 {
namespace seg {

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

using chunk::bf16;

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
    int P = 1;
    // double while the segment-sequences still fit in one wave and every
    // segment keeps at least 8 whole chunks
    while (seqs * P * 2 <= sms && T % (2 * P * chunk::C) == 0 && T / (2 * P) >= 8 * chunk::C) P *= 2;
    return P >= 4 ? P : 1;  // the three passes pay off from four segments on
}

size_t segments_ws_bytes(int B, int T, int H, int dk, int dv, int P) {
    return seg::carve(nullptr, B, T, H, dk, dv, P, nullptr);
}

cudaError_t launch_chunk_fwd_segments(const ChunkFwdArgs &a, int dk, int dv, int P, void *ws, cudaStream_t s) {
    seg::Carve c;
    seg::carve(ws, a.B, a.T, a.H, dk, dv, P, &c);
    const int Bp = a.B * P, Tp = a.T / P;
    const size_t wstride = (size_t)chunk::C * dk;
    cudaError_t e = cudaMemsetAsync(c.zeros, 0, (size_t)a.B * a.T * a.H * dk * sizeof(seg::bf16), s);
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
