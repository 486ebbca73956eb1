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

bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
// token rows of a batch: B * T, or T for a packed one
long long varlen_rows(const int *cu, int B, int T) { return cu ? (long long)T : (long long)B * T; }

// Test knobs (gdn2_debug_set): the device waits' iteration limit and a chunk
// of the tensor-memory forward whose hand-over arrival is withheld.
uint32_t g_wait_limit = 0;
int g_withhold_ready = -1;

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

int gdn2_debug_set(int knob, long long value) {
    switch (knob) {
        case GDN2_DEBUG_WAIT_LIMIT:
            if (value < 0 || value > 0xffffffffLL) return GDN2_ERR_INVALID_ARG;
            g_wait_limit = (uint32_t)value;
            return GDN2_OK;
        case GDN2_DEBUG_WITHHOLD_READY:
            if (value < -1 || value > 0x7fffffffLL) return GDN2_ERR_INVALID_ARG;
            g_withhold_ready = (int)value;
            return GDN2_OK;
        default: return GDN2_ERR_INVALID_ARG;
    }
}

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

}  // extern "C"

namespace {

// A scalar-gate tensor ([.., H], one element per token and head) needs only
// element alignment.
bool ok_gate(const void *p, int dtype) {
    return p != nullptr && (reinterpret_cast<uintptr_t>(p) & (dtype == GDN2_BF16 ? 1u : 3u)) == 0;
}

int decode_impl(const void *q, const void *k, const void *v, const void *log_alpha, const void *b, const void *w,
                float *S, void *o, int gates, int B, int H, int dk, int dv, int dtype, cudaStream_t stream) {
    int st = check_sizes(B, 1, H, dk, dv, dtype);
    if (st != GDN2_OK) return st;
    if (B == 0 || H == 0) return GDN2_OK;
    const bool la_ok = gates == kGatesGDN ? ok_gate(log_alpha, dtype) : ok_ptr(log_alpha);
    const bool bw_ok = gates == kGatesFull ? ok_ptr(b) && ok_ptr(w) : ok_gate(b, dtype);
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !la_ok || !bw_ok || !ok_ptr(S) || !ok_ptr(o))
        return GDN2_ERR_INVALID_ARG;
    RecurrentArgs a{q, k, v, log_alpha, b, w, S, S, o, B, 1, H};
    a.gates = gates;
    return launch_status(launch_recurrent_fwd(a, dk, dv, dtype == GDN2_BF16, stream));
}

}  // namespace

extern "C" {

int gdn2_decode_step(const void *q, const void *k, const void *v, const void *log_alpha,
                     const void *b, const void *w, float *S, void *o,
                     int B, int H, int dk, int dv, int dtype, cudaStream_t stream) {
    return decode_impl(q, k, v, log_alpha, b, w, S, o, kGatesFull, B, H, dk, dv, dtype, stream);
}

int gdn2_decode_step_kda(const void *q, const void *k, const void *v, const void *log_alpha, const void *beta,
                         float *S, void *o, int B, int H, int dk, int dv, int dtype, cudaStream_t stream) {
    return decode_impl(q, k, v, log_alpha, beta, beta, S, o, kGatesKDA, B, H, dk, dv, dtype, stream);
}

int gdn2_decode_step_gdn(const void *q, const void *k, const void *v, const void *log_alpha, const void *beta,
                         float *S, void *o, int B, int H, int dk, int dv, int dtype, cudaStream_t stream) {
    return decode_impl(q, k, v, log_alpha, beta, beta, S, o, kGatesGDN, B, H, dk, dv, dtype, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Chunk forward / backward for fixed-length batches (cu == nullptr: B
// sequences of T tokens) and packed variable-length batches (cu: B + 1 offsets
// into T token rows; see SeqView in launch.h).

namespace {

size_t fwd_ws_bytes(int B, int T, int H, int dk, int dv, int dtype, bool varlen) {
    if (check_sizes(B, T, H, dk, dv, dtype) != GDN2_OK) return 0;
    if (B == 0 || H == 0 || T == 0 || dtype != GDN2_BF16) return 0;
    const size_t plain = chunk_fwd_ws_bytes(B, H, dk);
    if (varlen) return plain;  // (packed batches always run one CTA per sequence)
    const int P = segment_count(B, T, H, dk, dv);
    if (P <= 1) return plain;
    size_t need = std::max(plain, segments_ws_bytes(B, T, H, dk, dv, P));
    const int Pt = seg_train_count(B, T, H, dk, dv);  // (the saving forward's segment path)
    if (Pt > 1) need = std::max(need, seg_train_fwd_ws_bytes(B, T, H, Pt));
    return need;
}

int fwd_impl(const void *q, const void *k, const void *v, const void *log_alpha, const void *b, const void *w,
             const float *S0, void *o, float *S_T, void *states, const int *cu, int B, int T, int H, int dk, int dv,
             int dtype, void *ws, size_t ws_bytes, cudaStream_t stream, int gates = kGatesFull,
             const void *out_gate = nullptr, const float *gamma = nullptr) {
    int st = check_sizes(B, T, H, dk, dv, dtype);
    if (st != GDN2_OK) return st;
    if (!ok_opt(S0) || !ok_opt(S_T) || !ok_opt(ws)) return GDN2_ERR_INVALID_ARG;
    if (cu && !aligned4(cu)) return GDN2_ERR_INVALID_ARG;
    if (B == 0 || H == 0) return GDN2_OK;
    if (T == 0) return copy_state(S_T, S0, B, H, dk, dv, stream);  // every sequence is empty
    // scalar gates run on the tensor-memory kernels (bf16, dk = dv = 128) or in fp32
    if (gates != kGatesFull && dtype == GDN2_BF16 && (dk != 128 || dv != 128)) return GDN2_ERR_UNSUPPORTED;
    const bool la_ok = gates == kGatesGDN ? ok_gate(log_alpha, dtype) : ok_ptr(log_alpha);
    const bool bw_ok = gates == kGatesFull ? ok_ptr(b) && ok_ptr(w) : ok_gate(b, dtype);
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !la_ok || !bw_ok || !ok_ptr(o)) return GDN2_ERR_INVALID_ARG;
    const bool keep = states != nullptr && dtype == GDN2_BF16;
    if (keep && !ok_ptr(states)) return GDN2_ERR_INVALID_ARG;
    // the one-CTA-per-sequence path needs the plain size; the workspace size
    // query's larger figure, where it applies, enables sequence segments
    const size_t need = dtype == GDN2_BF16 ? chunk_fwd_ws_bytes(B, H, dk) : 0;
    if (ws_bytes < need || (need > 0 && ws == nullptr)) return GDN2_ERR_WORKSPACE;
    if (dtype == GDN2_BF16) {
        const bool varlen = cu != nullptr;
        // few long sequences, states kept: segmented training (its buffer layout
        // follows from the sizes alone, so the backward always finds it)
        const int Pt = (keep && !varlen && gates == kGatesFull) ? seg_train_count(B, T, H, dk, dv) : 1;
        if (Pt > 1) {
            if (ws_bytes < seg_train_fwd_ws_bytes(B, T, H, Pt)) return GDN2_ERR_WORKSPACE;
            ChunkFwdArgs a{q, k, v, log_alpha, b, w, S0, o, S_T, nullptr, 0, nullptr, nullptr, nullptr,
                           status_ptr(), B, T, H};
            a.wait_limit = g_wait_limit;
            return launch_status(launch_seg_train_fwd(a, states, Pt, ws, stream));
        }
        char *sb = static_cast<char *>(states);
        ChunkFwdArgs a{q, k, v, log_alpha, b, w, S0, o, S_T, static_cast<float *>(ws), (size_t)64 * dk,
                       keep ? sb : nullptr,
                       keep ? sb + states_region_bytes(B, T, H, dk, dv, varlen) : nullptr,
                       keep ? sb + states_region_bytes(B, T, H, dk, dv, varlen) +
                                  intra_region_bytes(B, T, H, dv, varlen)
                            : nullptr,
                       status_ptr(), B, T, H, cu};
        a.gates = gates;
        a.wait_limit = g_wait_limit;
        a.withhold_ready = g_withhold_ready;
        bool segmented = false;
        if (!keep && !varlen && gates == kGatesFull) {
            const int P = segment_count(B, T, H, dk, dv);
            if (P > 1 && ws_bytes >= segments_ws_bytes(B, T, H, dk, dv, P)) {
                segmented = true;
                const int e = launch_status(launch_chunk_fwd_segments(a, dk, dv, P, ws, stream));
                if (e != GDN2_OK || !out_gate) return e;
            }
        }
        if (!segmented) {
            // the output epilogue runs inside the tensor-memory forward's O epilogue
            const bool fused = out_gate && !keep && dk == 128 && dv == 128;
            if (fused) {
                a.out_gate = out_gate;
                a.gamma = gamma;
            }
            const int e = launch_status(launch_chunk_fwd(a, dk, dv, stream));
            if (e != GDN2_OK || !out_gate || fused) return e;
        }
        // otherwise o first, then the epilogue on it in place
        return gdn2_output_gate_fwd(o, out_gate, gamma, o, (long long)(varlen ? T : (long long)B * T), H, dv, dtype,
                                    stream);
    }
    // fp32 precision mode: the recurrence token by token in fp32
    RecurrentArgs a{q, k, v, log_alpha, b, w, S0, S_T, o, B, T, H, cu};
    a.gates = gates;
    const int e = launch_status(launch_recurrent_fwd(a, dk, dv, false, stream));
    if (e != GDN2_OK || !out_gate) return e;
    return gdn2_output_gate_fwd(o, out_gate, gamma, o, (long long)(varlen_rows(cu, B, T)), H, dv, dtype, stream);
}

size_t bwd_ws_bytes(int B, int T, int H, int dk, int dv, int dtype, bool varlen) {
    if (check_sizes(B, T, H, dk, dv, dtype) != GDN2_OK) return 0;
    if (B == 0 || H == 0 || T == 0) return 0;
    if (dtype == GDN2_BF16) return chunk_bwd_ws_bytes(B, T, H, dk, dv, nullptr, nullptr, varlen);
    return recurrent_bwd_ws_bytes(B, T, H, dk, dv, varlen);
}

size_t states_bytes(int B, int T, int H, int dk, int dv, int dtype, bool varlen) {
    if (check_sizes(B, T, H, dk, dv, dtype) != GDN2_OK) return 0;
    if (B == 0 || H == 0 || T == 0 || dtype != GDN2_BF16) return 0;
    const int Pt = varlen ? 1 : seg_train_count(B, T, H, dk, dv);
    if (Pt > 1) return seg_train_states_bytes(B, T, H, Pt);
    size_t sbytes = 0;
    chunk_bwd_ws_bytes(B, T, H, dk, dv, nullptr, &sbytes, varlen);
    return sbytes;
}

size_t bwd_saved_ws_bytes(int B, int T, int H, int dk, int dv, int dtype, bool varlen) {
    if (check_sizes(B, T, H, dk, dv, dtype) != GDN2_OK) return 0;
    if (B == 0 || H == 0 || T == 0) return 0;
    if (dtype != GDN2_BF16) return bwd_ws_bytes(B, T, H, dk, dv, dtype, varlen);
    const int Pt = varlen ? 1 : seg_train_count(B, T, H, dk, dv);
    if (Pt > 1) return seg_train_bwd_ws_bytes(B, T, H, Pt);
    size_t sbytes = 0;
    return chunk_bwd_ws_bytes(B, T, H, dk, dv, nullptr, &sbytes, varlen) - sbytes;
}

// Shared body of the backward entry points (states == nullptr: the forward's
// chunk-boundary states and tiles are recomputed into the workspace).
int bwd_impl(const void *q, const void *k, const void *v, const void *log_alpha, const void *b, const void *w,
             const float *S0, const void *dO, const float *dS_T, const void *states, void *dq, void *dk_, void *dv_,
             void *dlog_alpha, void *db, void *dw, float *dS0, const int *cu, int B, int T, int H, int dk, int dv,
             int dtype, void *ws, size_t ws_bytes, cudaStream_t stream, int gates = kGatesFull) {
    int st = check_sizes(B, T, H, dk, dv, dtype);
    if (st != GDN2_OK) return st;
    if (!ok_opt(S0) || !ok_opt(dS_T) || !ok_opt(dS0) || !ok_opt(ws)) return GDN2_ERR_INVALID_ARG;
    if (cu && !aligned4(cu)) return GDN2_ERR_INVALID_ARG;
    if (B == 0 || H == 0) return GDN2_OK;
    if (T == 0) return copy_state(dS0, dS_T, B, H, dk, dv, stream);
    // scalar gates: the tensor-memory backward only (bf16, dk = dv = 128)
    if (gates != kGatesFull && (dtype != GDN2_BF16 || dk != 128 || dv != 128)) return GDN2_ERR_UNSUPPORTED;
    const bool la_ok = gates == kGatesGDN ? ok_gate(log_alpha, dtype) && ok_gate(dlog_alpha, dtype)
                                          : ok_ptr(log_alpha) && ok_ptr(dlog_alpha);
    const bool bw_ok = gates == kGatesFull ? ok_ptr(b) && ok_ptr(w) && ok_ptr(db) && ok_ptr(dw)
                                           : ok_gate(b, dtype) && ok_gate(db, dtype);
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !la_ok || !bw_ok || !ok_ptr(dO) || !ok_ptr(dq) || !ok_ptr(dk_) ||
        !ok_ptr(dv_))
        return GDN2_ERR_INVALID_ARG;
    const bool varlen = cu != nullptr;
    const bool saved = states != nullptr && dtype == GDN2_BF16;
    if (saved && !aligned16(states)) return GDN2_ERR_INVALID_ARG;
    const size_t need = saved ? bwd_saved_ws_bytes(B, T, H, dk, dv, dtype, varlen)
                              : bwd_ws_bytes(B, T, H, dk, dv, dtype, varlen);
    if (ws_bytes < need || (need > 0 && ws == nullptr)) return GDN2_ERR_WORKSPACE;
    if (dtype == GDN2_BF16) {
        const int Pt = (saved && !varlen && gates == kGatesFull) ? seg_train_count(B, T, H, dk, dv) : 1;
        if (Pt > 1) {  // segmented training: the forward kept its own layout
            ChunkBwdArgs a{q, k, v, log_alpha, b, w, S0, dO, dS_T, dq, dk_, dv_, dlog_alpha, db, dw, dS0, nullptr,
                           nullptr, nullptr, nullptr, 0, status_ptr(), 1, B, T, H};
            a.wait_limit = g_wait_limit;
            return launch_status(launch_seg_train_bwd(a, states, Pt, ws, stream));
        }
        size_t stride = 0, sbytes = 0;
        chunk_bwd_ws_bytes(B, T, H, dk, dv, &stride, &sbytes, varlen);
        char *st_buf = saved ? static_cast<char *>(const_cast<void *>(states)) : static_cast<char *>(ws);
        float *scr = reinterpret_cast<float *>(static_cast<char *>(ws) + (saved ? 0 : sbytes));
        const size_t rs = states_region_bytes(B, T, H, dk, dv, varlen);
        ChunkBwdArgs a{q, k, v, log_alpha, b, w, S0, dO, dS_T, dq, dk_, dv_, dlog_alpha, db, dw, dS0, st_buf,
                       st_buf + rs, st_buf + rs + intra_region_bytes(B, T, H, dv, varlen), scr, stride,
                       status_ptr(), saved ? 1 : 0, B, T, H, cu};
        a.gates = gates;
        a.wait_limit = g_wait_limit;
        return launch_status(launch_chunk_bwd(a, dk, dv, stream));
    }
    // fp32 precision mode: reverse-time recurrence token by token in fp32
    RecurrentBwdArgs a{q, k, v, log_alpha, b, w, S0, dO, dS_T, dq, dk_, dv_, dlog_alpha, db, dw,
                       dS0, static_cast<float *>(ws), B, T, H, cu};
    return launch_status(launch_recurrent_bwd(a, dk, dv, false, stream));
}

}  // namespace

extern "C" {

size_t gdn2_chunk_fwd_workspace(int B, int T, int H, int dk, int dv, int dtype) {
    return fwd_ws_bytes(B, T, H, dk, dv, dtype, false);
}

int gdn2_chunk_fwd(const void *q, const void *k, const void *v, const void *log_alpha,
                   const void *b, const void *w, const float *S0, void *o, float *S_T,
                   int B, int T, int H, int dk, int dv, int dtype,
                   void *ws, size_t ws_bytes, cudaStream_t stream) {
    return fwd_impl(q, k, v, log_alpha, b, w, S0, o, S_T, nullptr, nullptr, B, T, H, dk, dv, dtype, ws, ws_bytes,
                    stream);
}

size_t gdn2_chunk_bwd_workspace(int B, int T, int H, int dk, int dv, int dtype) {
    return bwd_ws_bytes(B, T, H, dk, dv, dtype, false);
}

int gdn2_chunk_bwd(const void *q, const void *k, const void *v, const void *log_alpha,
                   const void *b, const void *w, const float *S0, const void *dO,
                   const float *dS_T, void *dq, void *dk_, void *dv_, void *dlog_alpha,
                   void *db, void *dw, float *dS0,
                   int B, int T, int H, int dk, int dv, int dtype,
                   void *ws, size_t ws_bytes, cudaStream_t stream) {
    return bwd_impl(q, k, v, log_alpha, b, w, S0, dO, dS_T, nullptr, dq, dk_, dv_, dlog_alpha, db, dw, dS0, nullptr,
                    B, T, H, dk, dv, dtype, ws, ws_bytes, stream);
}

size_t gdn2_chunk_states_bytes(int B, int T, int H, int dk, int dv, int dtype) {
    return states_bytes(B, T, H, dk, dv, dtype, false);
}

int gdn2_chunk_fwd_save(const void *q, const void *k, const void *v, const void *log_alpha,
                        const void *b, const void *w, const float *S0, void *o, float *S_T, void *states,
                        int B, int T, int H, int dk, int dv, int dtype,
                        void *ws, size_t ws_bytes, cudaStream_t stream) {
    if (dtype == GDN2_BF16 && B > 0 && H > 0 && T > 0 && states == nullptr) return GDN2_ERR_INVALID_ARG;
    return fwd_impl(q, k, v, log_alpha, b, w, S0, o, S_T, states, nullptr, B, T, H, dk, dv, dtype, ws, ws_bytes,
                    stream);
}

size_t gdn2_chunk_bwd_saved_workspace(int B, int T, int H, int dk, int dv, int dtype) {
    return bwd_saved_ws_bytes(B, T, H, dk, dv, dtype, false);
}

int gdn2_chunk_bwd_saved(const void *q, const void *k, const void *v, const void *log_alpha,
                         const void *b, const void *w, const float *S0, const void *dO,
                         const float *dS_T, const void *states, void *dq, void *dk_, void *dv_,
                         void *dlog_alpha, void *db, void *dw, float *dS0,
                         int B, int T, int H, int dk, int dv, int dtype,
                         void *ws, size_t ws_bytes, cudaStream_t stream) {
    if (dtype == GDN2_BF16 && B > 0 && H > 0 && T > 0 && states == nullptr) return GDN2_ERR_INVALID_ARG;
    return bwd_impl(q, k, v, log_alpha, b, w, S0, dO, dS_T, states, dq, dk_, dv_, dlog_alpha, db, dw, dS0, nullptr,
                    B, T, H, dk, dv, dtype, ws, ws_bytes, stream);
}

// ---- packed variable-length batches

size_t gdn2_chunk_fwd_varlen_workspace(int N, int total_T, int H, int dk, int dv, int dtype) {
    return fwd_ws_bytes(N, total_T, H, dk, dv, dtype, true);
}

int gdn2_chunk_fwd_varlen(const void *q, const void *k, const void *v, const void *log_alpha, const void *b,
                          const void *w, const float *S0, void *o, float *S_T, const int *cu_seqlens, int N,
                          int total_T, int H, int dk, int dv, int dtype, void *ws, size_t ws_bytes,
                          cudaStream_t stream) {
    if (cu_seqlens == nullptr) return GDN2_ERR_INVALID_ARG;
    return fwd_impl(q, k, v, log_alpha, b, w, S0, o, S_T, nullptr, cu_seqlens, N, total_T, H, dk, dv, dtype, ws,
                    ws_bytes, stream);
}

size_t gdn2_chunk_bwd_varlen_workspace(int N, int total_T, int H, int dk, int dv, int dtype) {
    return bwd_ws_bytes(N, total_T, H, dk, dv, dtype, true);
}

int gdn2_chunk_bwd_varlen(const void *q, const void *k, const void *v, const void *log_alpha, const void *b,
                          const void *w, const float *S0, const void *dO, const float *dS_T, void *dq, void *dk_,
                          void *dv_, void *dlog_alpha, void *db, void *dw, float *dS0, const int *cu_seqlens, int N,
                          int total_T, int H, int dk, int dv, int dtype, void *ws, size_t ws_bytes,
                          cudaStream_t stream) {
    if (cu_seqlens == nullptr) return GDN2_ERR_INVALID_ARG;
    return bwd_impl(q, k, v, log_alpha, b, w, S0, dO, dS_T, nullptr, dq, dk_, dv_, dlog_alpha, db, dw, dS0,
                    cu_seqlens, N, total_T, H, dk, dv, dtype, ws, ws_bytes, stream);
}

size_t gdn2_chunk_states_varlen_bytes(int N, int total_T, int H, int dk, int dv, int dtype) {
    return states_bytes(N, total_T, H, dk, dv, dtype, true);
}

int gdn2_chunk_fwd_save_varlen(const void *q, const void *k, const void *v, const void *log_alpha, const void *b,
                               const void *w, const float *S0, void *o, float *S_T, void *states,
                               const int *cu_seqlens, int N, int total_T, int H, int dk, int dv, int dtype,
                               void *ws, size_t ws_bytes, cudaStream_t stream) {
    if (cu_seqlens == nullptr) return GDN2_ERR_INVALID_ARG;
    if (dtype == GDN2_BF16 && N > 0 && H > 0 && total_T > 0 && states == nullptr) return GDN2_ERR_INVALID_ARG;
    return fwd_impl(q, k, v, log_alpha, b, w, S0, o, S_T, states, cu_seqlens, N, total_T, H, dk, dv, dtype, ws,
                    ws_bytes, stream);
}

size_t gdn2_chunk_bwd_saved_varlen_workspace(int N, int total_T, int H, int dk, int dv, int dtype) {
    return bwd_saved_ws_bytes(N, total_T, H, dk, dv, dtype, true);
}

int gdn2_chunk_bwd_saved_varlen(const void *q, const void *k, const void *v, const void *log_alpha, const void *b,
                                const void *w, const float *S0, const void *dO, const float *dS_T,
                                const void *states, void *dq, void *dk_, void *dv_, void *dlog_alpha, void *db,
                                void *dw, float *dS0, const int *cu_seqlens, int N, int total_T, int H, int dk,
                                int dv, int dtype, void *ws, size_t ws_bytes, cudaStream_t stream) {
    if (cu_seqlens == nullptr) return GDN2_ERR_INVALID_ARG;
    if (dtype == GDN2_BF16 && N > 0 && H > 0 && total_T > 0 && states == nullptr) return GDN2_ERR_INVALID_ARG;
    return bwd_impl(q, k, v, log_alpha, b, w, S0, dO, dS_T, states, dq, dk_, dv_, dlog_alpha, db, dw, dS0,
                    cu_seqlens, N, total_T, H, dk, dv, dtype, ws, ws_bytes, stream);
}

// ---- reduced gates: KDA (one scalar beta per token and head for both gates)
// and Gated DeltaNet (that, and a scalar decay)

int gdn2_chunk_fwd_kda(const void *q, const void *k, const void *v, const void *log_alpha, const void *beta,
                       const float *S0, void *o, float *S_T, int B, int T, int H, int dk, int dv, int dtype,
                       void *ws, size_t ws_bytes, cudaStream_t stream) {
    return fwd_impl(q, k, v, log_alpha, beta, beta, S0, o, S_T, nullptr, nullptr, B, T, H, dk, dv, dtype, ws,
                    ws_bytes, stream, kGatesKDA);
}

int gdn2_chunk_fwd_gdn(const void *q, const void *k, const void *v, const void *log_alpha, const void *beta,
                       const float *S0, void *o, float *S_T, int B, int T, int H, int dk, int dv, int dtype,
                       void *ws, size_t ws_bytes, cudaStream_t stream) {
    return fwd_impl(q, k, v, log_alpha, beta, beta, S0, o, S_T, nullptr, nullptr, B, T, H, dk, dv, dtype, ws,
                    ws_bytes, stream, kGatesGDN);
}

int gdn2_chunk_bwd_kda(const void *q, const void *k, const void *v, const void *log_alpha, const void *beta,
                       const float *S0, const void *dO, const float *dS_T, void *dq, void *dk_, void *dv_,
                       void *dlog_alpha, void *dbeta, float *dS0, int B, int T, int H, int dk, int dv, int dtype,
                       void *ws, size_t ws_bytes, cudaStream_t stream) {
    return bwd_impl(q, k, v, log_alpha, beta, beta, S0, dO, dS_T, nullptr, dq, dk_, dv_, dlog_alpha, dbeta, nullptr,
                    dS0, nullptr, B, T, H, dk, dv, dtype, ws, ws_bytes, stream, kGatesKDA);
}

int gdn2_chunk_bwd_gdn(const void *q, const void *k, const void *v, const void *log_alpha, const void *beta,
                       const float *S0, const void *dO, const float *dS_T, void *dq, void *dk_, void *dv_,
                       void *dlog_alpha, void *dbeta, float *dS0, int B, int T, int H, int dk, int dv, int dtype,
                       void *ws, size_t ws_bytes, cudaStream_t stream) {
    return bwd_impl(q, k, v, log_alpha, beta, beta, S0, dO, dS_T, nullptr, dq, dk_, dv_, dlog_alpha, dbeta, nullptr,
                    dS0, nullptr, B, T, H, dk, dv, dtype, ws, ws_bytes, stream, kGatesGDN);
}

// ---- the forward with the output epilogue: z = o / rms(o) * gamma * silu(g)

int gdn2_chunk_fwd_gated(const void *q, const void *k, const void *v, const void *log_alpha, const void *b,
                         const void *w, const float *S0, const void *g, const float *gamma, void *z, float *S_T, int B,
                         int T, int H, int dk, int dv, int dtype, void *ws, size_t ws_bytes, cudaStream_t stream) {
    if (B > 0 && H > 0 && T > 0 && (!ok_ptr(g) || !ok_ptr(gamma))) return GDN2_ERR_INVALID_ARG;
    return fwd_impl(q, k, v, log_alpha, b, w, S0, z, S_T, nullptr, nullptr, B, T, H, dk, dv, dtype, ws, ws_bytes,
                    stream, kGatesFull, g, gamma);
}

}  // extern "C"
