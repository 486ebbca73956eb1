// C ABI of the GDN-2 mixer: host-side argument checks, workspace sizing,
// dispatch to the sm_100a kernels and the device status word.  Declarations
// and the contract of every entry point are in include/gdn2.h.
#include "gdn2.h"

#include <stdint.h>

#include <algorithm>

#include "launch.h"

namespace gdn2 {

// Library-owned device status word: one per device that loads the library.
__device__ int g_device_status = 0;

namespace {

constexpr int kMaxDevices = 64;
int *g_status_ptr[kMaxDevices] = {nullptr};

// Device address of the status word on the current device (nullptr on failure).
int *status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    if (!g_status_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = static_cast<int *>(p);
    }
    return g_status_ptr[dev];
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_ptr(const void *p) { return p != nullptr && aligned16(p); }
bool ok_opt(const void *p) { return p == nullptr || aligned16(p); }
bool ok_dim(int d) { return d == 64 || d == 128; }

int check_sizes(int B, int T, int H, int dk, int dv, int dtype) {
    if (B < 0 || T < 0 || H < 0) return GDN2_ERR_INVALID_ARG;
    if (dtype != GDN2_BF16 && dtype != GDN2_FP32) return GDN2_ERR_UNSUPPORTED;
    if (!ok_dim(dk) || !ok_dim(dv)) return GDN2_ERR_UNSUPPORTED;
    if ((long long)B * H > 0x7fffffffLL) return GDN2_ERR_INVALID_ARG;
    return GDN2_OK;
}

int launch_status(cudaError_t e) {
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return GDN2_ERR_CUDA;
    }
    return GDN2_OK;
}

// Copy S0 (or zeros) into a state buffer of B*H*dk*dv floats.
int copy_state(float *dst, const float *src, int B, int H, int dk, int dv, cudaStream_t s) {
    if (!dst) return GDN2_OK;
    const size_t bytes = (size_t)B * H * dk * dv * sizeof(float);
    cudaError_t e = src ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, s)
                        : cudaMemsetAsync(dst, 0, bytes, s);
    return launch_status(e);
}

}  // namespace
}  // namespace gdn2

using namespace gdn2;

extern "C" {

int gdn2_version(void) { return 100; }

const char *gdn2_status_string(int status) {
    switch (status) {
        case GDN2_OK: return "GDN2_OK";
        case GDN2_ERR_INVALID_ARG: return "GDN2_ERR_INVALID_ARG: null, misaligned or out-of-range argument";
        case GDN2_ERR_UNSUPPORTED: return "GDN2_ERR_UNSUPPORTED: dk/dv must be 64 or 128; dtype GDN2_BF16 or GDN2_FP32";
        case GDN2_ERR_CUDA: return "GDN2_ERR_CUDA: a CUDA call or kernel launch failed";
        case GDN2_ERR_TIMEOUT: return "GDN2_ERR_TIMEOUT: a bounded device-side wait ran out";
        case GDN2_ERR_WORKSPACE: return "GDN2_ERR_WORKSPACE: workspace missing or too small";
        default: return "GDN2: unknown status";
    }
}

int gdn2_get_device_status(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) {
        (void)cudaGetLastError();
        return GDN2_ERR_CUDA;
    }
    int *p = status_ptr();
    if (!p) return GDN2_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return GDN2_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return GDN2_ERR_CUDA;
    }
    return v;
}

size_t gdn2_chunk_fwd_workspace(int B, int T, int H, int dk, int dv, int dtype) {
    if (check_sizes(B, T, H, dk, dv, dtype) != GDN2_OK) return 0;
    if (B == 0 || H == 0 || T == 0 || dtype != GDN2_BF16) return 0;
    const size_t plain = chunk_fwd_ws_bytes(B, H, dk);
    const int P = segment_count(B, T, H, dk, dv);
    return P > 1 ? std::max(plain, segments_ws_bytes(B, T, H, dk, dv, P)) : plain;
}

int gdn2_chunk_fwd(const void *q, const void *k, const void *v, const void *log_alpha,
                   const void *b, const void *w, const float *S0, void *o, float *S_T,
                   int B, int T, int H, int dk, int dv, int dtype,
                   void *ws, size_t ws_bytes, cudaStream_t stream) {
    int st = check_sizes(B, T, H, dk, dv, dtype);
    if (st != GDN2_OK) return st;
    if (!ok_opt(S0) || !ok_opt(S_T) || !ok_opt(ws)) return GDN2_ERR_INVALID_ARG;
    if (B == 0 || H == 0) return GDN2_OK;
    if (T == 0) return copy_state(S_T, S0, B, H, dk, dv, stream);
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(log_alpha) || !ok_ptr(b) || !ok_ptr(w) ||
        !ok_ptr(o))
        return GDN2_ERR_INVALID_ARG;
    // the one-CTA-per-sequence path needs the plain size; the workspace size
    // query's larger figure, where it applies, enables sequence segments
    const size_t need = dtype == GDN2_BF16 ? chunk_fwd_ws_bytes(B, H, dk) : 0;
    if (ws_bytes < need || (need > 0 && ws == nullptr)) return GDN2_ERR_WORKSPACE;
    if (dtype == GDN2_BF16) {
        ChunkFwdArgs a{q, k, v, log_alpha, b, w, S0, o, S_T, static_cast<float *>(ws),
                       (size_t)64 * dk, nullptr, nullptr, nullptr, status_ptr(), B, T, H};
        const int P = segment_count(B, T, H, dk, dv);
        if (P > 1 && ws_bytes >= segments_ws_bytes(B, T, H, dk, dv, P))
            return launch_status(launch_chunk_fwd_segments(a, dk, dv, P, ws, stream));
        return launch_status(launch_chunk_fwd(a, dk, dv, stream));
    }
    // fp32 precision mode: the recurrence token by token in fp32
    RecurrentArgs a{q, k, v, log_alpha, b, w, S0, S_T, o, B, T, H};
    return launch_status(launch_recurrent_fwd(a, dk, dv, false, stream));
}

int gdn2_decode_step(const void *q, const void *k, const void *v, const void *log_alpha,
                     const void *b, const void *w, float *S, void *o,
                     int B, int H, int dk, int dv, int dtype, cudaStream_t stream) {
    int st = check_sizes(B, 1, H, dk, dv, dtype);
    if (st != GDN2_OK) return st;
    if (B == 0 || H == 0) return GDN2_OK;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(log_alpha) || !ok_ptr(b) || !ok_ptr(w) ||
        !ok_ptr(S) || !ok_ptr(o))
        return GDN2_ERR_INVALID_ARG;
    RecurrentArgs a{q, k, v, log_alpha, b, w, S, S, o, B, 1, H};
    return launch_status(launch_recurrent_fwd(a, dk, dv, dtype == GDN2_BF16, stream));
}

size_t gdn2_chunk_bwd_workspace(int B, int T, int H, int dk, int dv, int dtype) {
    if (check_sizes(B, T, H, dk, dv, dtype) != GDN2_OK) return 0;
    if (B == 0 || H == 0 || T == 0) return 0;
    if (dtype == GDN2_BF16) return chunk_bwd_ws_bytes(B, T, H, dk, dv, nullptr, nullptr);
    return recurrent_bwd_ws_bytes(B, T, H, dk, dv);
}

}  // extern "C"

namespace {

// Shared body of gdn2_chunk_bwd (states == nullptr: recomputed into the
// workspace) and gdn2_chunk_bwd_saved (states from gdn2_chunk_fwd_save).
int chunk_bwd_impl(const void *q, const void *k, const void *v, const void *log_alpha, const void *b,
                   const void *w, const float *S0, const void *dO, const float *dS_T, const void *states,
                   void *dq, void *dk_, void *dv_, void *dlog_alpha, void *db, void *dw, float *dS0, int B, int T,
                   int H, int dk, int dv, int dtype, void *ws, size_t ws_bytes, cudaStream_t stream) {
    int st = check_sizes(B, T, H, dk, dv, dtype);
    if (st != GDN2_OK) return st;
    if (!ok_opt(S0) || !ok_opt(dS_T) || !ok_opt(dS0) || !ok_opt(ws)) return GDN2_ERR_INVALID_ARG;
    if (B == 0 || H == 0) return GDN2_OK;
    if (T == 0) return copy_state(dS0, dS_T, B, H, dk, dv, stream);
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(log_alpha) || !ok_ptr(b) || !ok_ptr(w) ||
        !ok_ptr(dO) || !ok_ptr(dq) || !ok_ptr(dk_) || !ok_ptr(dv_) || !ok_ptr(dlog_alpha) ||
        !ok_ptr(db) || !ok_ptr(dw))
        return GDN2_ERR_INVALID_ARG;
    const bool saved = states != nullptr && dtype == GDN2_BF16;
    if (saved && !aligned16(states)) return GDN2_ERR_INVALID_ARG;
    const size_t need = saved ? gdn2_chunk_bwd_saved_workspace(B, T, H, dk, dv, dtype)
                              : gdn2_chunk_bwd_workspace(B, T, H, dk, dv, dtype);
    if (ws_bytes < need || (need > 0 && ws == nullptr)) return GDN2_ERR_WORKSPACE;
    if (dtype == GDN2_BF16) {
        size_t stride = 0, sbytes = 0;
        chunk_bwd_ws_bytes(B, T, H, dk, dv, &stride, &sbytes);
        char *st_buf = saved ? static_cast<char *>(const_cast<void *>(states)) : static_cast<char *>(ws);
        float *scr = reinterpret_cast<float *>(static_cast<char *>(ws) + (saved ? 0 : sbytes));
        ChunkBwdArgs a{q, k, v, log_alpha, b, w, S0, dO, dS_T, dq, dk_, dv_, dlog_alpha, db, dw, dS0, st_buf,
                       st_buf + states_region_bytes(B, T, H, dk, dv),
                       st_buf + states_region_bytes(B, T, H, dk, dv) + intra_region_bytes(B, T, H, dv), scr, stride,
                       status_ptr(), saved ? 1 : 0,
                       B, T, H};
        return launch_status(launch_chunk_bwd(a, dk, dv, stream));
    }
    // fp32 precision mode: reverse-time recurrence token by token in fp32
    RecurrentBwdArgs a{q, k, v, log_alpha, b, w, S0, dO, dS_T, dq, dk_, dv_, dlog_alpha, db, dw,
                       dS0, static_cast<float *>(ws), B, T, H};
    return launch_status(launch_recurrent_bwd(a, dk, dv, false, stream));
}

}  // namespace

extern "C" {

int gdn2_chunk_bwd(const void *q, const void *k, const void *v, const void *log_alpha,
                   const void *b, const void *w, const float *S0, const void *dO,
                   const float *dS_T, void *dq, void *dk_, void *dv_, void *dlog_alpha,
                   void *db, void *dw, float *dS0,
                   int B, int T, int H, int dk, int dv, int dtype,
                   void *ws, size_t ws_bytes, cudaStream_t stream) {
    return chunk_bwd_impl(q, k, v, log_alpha, b, w, S0, dO, dS_T, nullptr, dq, dk_, dv_, dlog_alpha, db, dw, dS0,
                          B, T, H, dk, dv, dtype, ws, ws_bytes, stream);
}

size_t gdn2_chunk_states_bytes(int B, int T, int H, int dk, int dv, int dtype) {
    if (check_sizes(B, T, H, dk, dv, dtype) != GDN2_OK) return 0;
    if (B == 0 || H == 0 || T == 0 || dtype != GDN2_BF16) return 0;
    size_t sbytes = 0;
    chunk_bwd_ws_bytes(B, T, H, dk, dv, nullptr, &sbytes);
    return sbytes;
}

int gdn2_chunk_fwd_save(const void *q, const void *k, const void *v, const void *log_alpha,
                        const void *b, const void *w, const float *S0, void *o, float *S_T, void *states,
                        int B, int T, int H, int dk, int dv, int dtype,
                        void *ws, size_t ws_bytes, cudaStream_t stream) {
    int st = check_sizes(B, T, H, dk, dv, dtype);
    if (st != GDN2_OK) return st;
    if (dtype != GDN2_BF16 || B == 0 || H == 0 || T == 0)
        return gdn2_chunk_fwd(q, k, v, log_alpha, b, w, S0, o, S_T, B, T, H, dk, dv, dtype, ws, ws_bytes, stream);
    if (!ok_opt(S0) || !ok_opt(S_T) || !ok_opt(ws) || !ok_ptr(states)) return GDN2_ERR_INVALID_ARG;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(log_alpha) || !ok_ptr(b) || !ok_ptr(w) ||
        !ok_ptr(o))
        return GDN2_ERR_INVALID_ARG;
    const size_t need = chunk_fwd_ws_bytes(B, H, dk);  // (the training forward is never segmented)
    if (ws_bytes < need || (need > 0 && ws == nullptr)) return GDN2_ERR_WORKSPACE;
    ChunkFwdArgs a{q, k, v, log_alpha, b, w, S0, o, S_T, static_cast<float *>(ws), (size_t)64 * dk, states,
                   static_cast<char *>(states) + states_region_bytes(B, T, H, dk, dv),
                   static_cast<char *>(states) + states_region_bytes(B, T, H, dk, dv) + intra_region_bytes(B, T, H, dv),
                   status_ptr(), B, T, H};
    return launch_status(launch_chunk_fwd(a, dk, dv, stream));
}

size_t gdn2_chunk_bwd_saved_workspace(int B, int T, int H, int dk, int dv, int dtype) {
    if (check_sizes(B, T, H, dk, dv, dtype) != GDN2_OK) return 0;
    if (B == 0 || H == 0 || T == 0) return 0;
    if (dtype != GDN2_BF16) return gdn2_chunk_bwd_workspace(B, T, H, dk, dv, dtype);
    size_t sbytes = 0;
    return chunk_bwd_ws_bytes(B, T, H, dk, dv, nullptr, &sbytes) - sbytes;
}

int gdn2_chunk_bwd_saved(const void *q, const void *k, const void *v, const void *log_alpha,
                         const void *b, const void *w, const float *S0, const void *dO,
                         const float *dS_T, const void *states, void *dq, void *dk_, void *dv_,
                         void *dlog_alpha, void *db, void *dw, float *dS0,
                         int B, int T, int H, int dk, int dv, int dtype,
                         void *ws, size_t ws_bytes, cudaStream_t stream) {
    if (dtype == GDN2_BF16 && B > 0 && H > 0 && T > 0 && states == nullptr) return GDN2_ERR_INVALID_ARG;
    return chunk_bwd_impl(q, k, v, log_alpha, b, w, S0, dO, dS_T, states, dq, dk_, dv_, dlog_alpha, db, dw, dS0,
                          B, T, H, dk, dv, dtype, ws, ws_bytes, stream);
}

}  // extern "C"
