/*
 * gdn2.h -- C ABI of the B200 (sm_100a) Gated DeltaNet-2 sequence mixer.
 *
 * The operation: per batch b and head h, a state S in R^{dk x dv} (rows = key
 * channels, columns = value channels) evolves token by token as
 *
 *     S_t = (I - k_t (b_t . k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t . v_t)^T
 *     o_t = S_t^T q_t
 *
 * ("Why NVIDIA Gated DeltaNet-2 separates erase and write gates", axbrief,
 * section "Gated Delta Rule-2: per-channel erase/write split": the recurrence,
 * the per-key-channel decay alpha_t = exp(log_alpha_t), the erase gate
 * b_t in [0,1]^dk on the key axis and the write gate w_t in [0,1]^dv on the
 * value axis; the readout o_t = S_t^T q_t after the update is this library's
 * reading, the pages leave it open.)  The same section fixes the chunk size
 * C = 64 of the chunk-parallel form and asks for a backward pass whose gate
 * factors sit inside every gradient-accumulating inner product.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every tensor pointer is a DEVICE pointer to a caller-owned buffer.  The
 *   library never allocates or frees memory and never synchronises the
 *   stream, except gdn2_get_device_status().  All work is enqueued on the
 *   caller's stream `stream` (0 = legacy default stream).
 * - Token tensors (q, k, log_alpha, b: last dim dk; v, w, o, dO: last dim dv)
 *   are [B, T, H, D] contiguous (D fastest) for the chunk calls and [B, H, D]
 *   for the decode step, in the element type given by `dtype`.  Gradients
 *   have the shape and dtype of their input.
 * - States (S0, S_T, S, dS_T, dS0) are fp32 [B, H, dk, dv] row-major.
 * - Every pointer must be 16-byte aligned.  dk, dv in {64, 128}.
 * - Preconditions the library does not check on the device: q and k are
 *   already L2-normalised by the caller (the q/k path ends in an L2 norm on
 *   the pages); log_alpha <= 0 (any finite value, large negative = reset);
 *   b, w in [0, 1]; no output aliases an input (except S in the decode step).
 * - Return value: GDN2_OK (0) or a negative gdn2_status.  Arguments are
 *   checked on the host BEFORE anything is launched; on an error nothing is
 *   enqueued.  A launch failure returns GDN2_ERR_CUDA.  Errors that happen on
 *   the device (a bounded wait that ran out) are recorded in a library-owned
 *   device status word that gdn2_get_device_status() reads and clears.
 * - Results are deterministic: no atomics take part in any reduction.
 */
#ifndef GDN2_H
#define GDN2_H

#include <stddef.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDN2_OK = 0,
    GDN2_ERR_INVALID_ARG = -1,  /* null pointer, bad size, misaligned pointer */
    GDN2_ERR_UNSUPPORTED = -2,  /* dk or dv outside {64, 128}, unknown dtype */
    GDN2_ERR_CUDA = -3,         /* a CUDA runtime call or launch failed */
    GDN2_ERR_TIMEOUT = -4,      /* a device-side bounded wait ran out */
    GDN2_ERR_WORKSPACE = -5     /* workspace missing or smaller than required */
} gdn2_status;

typedef enum {
    GDN2_BF16 = 0,  /* token tensors in bfloat16; chunk path on tensor cores */
    GDN2_FP32 = 1   /* token tensors in fp32; fp32 arithmetic throughout */
} gdn2_dtype;

/*
 * Bytes of device workspace for gdn2_chunk_fwd at these sizes (may be 0).
 * For bf16 with dk = dv and too few sequences to fill the GPU (B*H*4 <= the
 * SM count) with T a multiple of 4 segments of at least 8 chunks, this is the
 * size of the sequence-segmented forward (below); otherwise, and always for
 * fp32, it is the one-CTA-per-sequence forward's B*H*64*dk*4 bytes.
 */
size_t gdn2_chunk_fwd_workspace(int B, int T, int H, int dk, int dv, int dtype);

/*
 * Chunk-parallel forward over T tokens (chunks of C = 64 tokens; T need not
 * be a multiple of 64).  Computes o [B,T,H,dv] and, when S_T is non-null, the
 * final state S_T [B,H,dk,dv].  S0 may be null (zero initial state).
 * T = 0 is valid: it copies S0 (or zeros) to S_T.  B = 0 or H = 0 is a no-op.
 * ws/ws_bytes: caller-owned device workspace of at least B*H*64*dk*4 bytes
 * for bf16 (0 for fp32); ws may be null when that is 0.
 * With ws_bytes >= gdn2_chunk_fwd_workspace(...) where that figure is the
 * segmented one, each sequence runs as P equal segments side by side
 * (P = 4..16, up to the SM count): the state update of a chunk is affine in
 * the state (Gated Delta Rule-2 section of "Why NVIDIA Gated DeltaNet-2
 * separates erase and write gates"), so every segment's local end state and
 * dk x dk transition come from two forwards over the segments, an fp32 scan
 * over the segments gives their start states, and a third forward gives o and
 * S_T.  Same results to bf16 rounding; about three forwards of work on P times
 * as many SMs.
 */
int gdn2_chunk_fwd(const void *q, const void *k, const void *v, const void *log_alpha,
                   const void *b, const void *w, const float *S0, void *o, float *S_T,
                   int B, int T, int H, int dk, int dv, int dtype,
                   void *ws, size_t ws_bytes, cudaStream_t stream);

/*
 * One decode step (the same recurrence for a single token per sequence):
 * tokens [B,H,D], state S [B,H,dk,dv] fp32 updated IN PLACE, output o
 * [B,H,dv].  Each state is read once and written once.
 */
int gdn2_decode_step(const void *q, const void *k, const void *v, const void *log_alpha,
                     const void *b, const void *w, float *S, void *o,
                     int B, int H, int dk, int dv, int dtype, cudaStream_t stream);

/* Bytes of device workspace gdn2_chunk_bwd needs for these sizes. */
size_t gdn2_chunk_bwd_workspace(int B, int T, int H, int dk, int dv, int dtype);

/*
 * Gate-aware backward (vector-Jacobian product) of gdn2_chunk_fwd: given the
 * forward inputs, the upstream gradient dO [B,T,H,dv] of o and dS_T of S_T
 * (null = zero), writes dq, dk_, dlog_alpha, db ([B,T,H,dk]), dv_, dw
 * ([B,T,H,dv]) and, when non-null, dS0 [B,H,dk,dv] fp32.  S0 may be null
 * (zero).  dlog_alpha is the gradient with respect to log_alpha; db and dw
 * with respect to the gates as passed (after any sigmoid).  Needs
 * gdn2_chunk_bwd_workspace(...) bytes of caller-owned device workspace.
 */
int gdn2_chunk_bwd(const void *q, const void *k, const void *v, const void *log_alpha,
                   const void *b, const void *w, const float *S0, const void *dO,
                   const float *dS_T, void *dq, void *dk_, void *dv_, void *dlog_alpha,
                   void *db, void *dw, float *dS0,
                   int B, int T, int H, int dk, int dv, int dtype,
                   void *ws, size_t ws_bytes, cudaStream_t stream);

/*
 * Saved-state training path.  gdn2_chunk_fwd_save is gdn2_chunk_fwd that
 * also keeps, in `states` (gdn2_chunk_states_bytes(...) bytes, caller-owned,
 * 16-byte aligned, contents private to this library), what the backward
 * needs from the forward: the state at every chunk boundary (bf16,
 * [B][H][ceil(T/64)+1][dk][dv]) and, per chunk, the bf16 WY factor
 * T = (I + A)^{-1}, the decayed query-key Gram M (64 x 64 each) and the
 * chunk's WY-form write U (64 x dv), and for dk = dv = 128 also the decayed
 * operands Qt, Gt, Kb (64 x 128 each).  gdn2_chunk_bwd_saved is gdn2_chunk_bwd
 * that reads these instead of re-running the forward to recompute them, with
 * the smaller workspace gdn2_chunk_bwd_saved_workspace(...).  The buffer must
 * come from gdn2_chunk_fwd_save on the same inputs; results equal those of
 * gdn2_chunk_fwd / gdn2_chunk_bwd bit for bit.  (The backward of the pages'
 * method needs the chunk-start states and these per-chunk products; this pair
 * keeps them instead of recomputing them.)
 * For GDN2_FP32 the state buffer is not used (gdn2_chunk_states_bytes = 0):
 * the fp32 mode checkpoints inside its own workspace.
 */
size_t gdn2_chunk_states_bytes(int B, int T, int H, int dk, int dv, int dtype);
int gdn2_chunk_fwd_save(const void *q, const void *k, const void *v, const void *log_alpha,
                        const void *b, const void *w, const float *S0, void *o, float *S_T, void *states,
                        int B, int T, int H, int dk, int dv, int dtype,
                        void *ws, size_t ws_bytes, cudaStream_t stream);
size_t gdn2_chunk_bwd_saved_workspace(int B, int T, int H, int dk, int dv, int dtype);
int gdn2_chunk_bwd_saved(const void *q, const void *k, const void *v, const void *log_alpha,
                         const void *b, const void *w, const float *S0, const void *dO,
                         const float *dS_T, const void *states, void *dq, void *dk_, void *dv_,
                         void *dlog_alpha, void *db, void *dw, float *dS0,
                         int B, int T, int H, int dk, int dv, int dtype,
                         void *ws, size_t ws_bytes, cudaStream_t stream);

/*
 * gdn2_chunk_fwd without a caller-provided workspace, for callers that cannot
 * allocate device memory (no cudaMalloc available to them, or a code path
 * that must not allocate).  The pages have no counterpart to this call; it is
 * an interface convenience of this library.
 *
 * Arguments, layouts, results and error codes are those of gdn2_chunk_fwd.
 * The scratch comes from an 8 MiB array in the library's device image, which
 * every GPU that loads the library holds until the process exits; problems
 * needing more (B*H*dk > 32768, e.g. B*H > 256 at dk = 128) get
 * GDN2_ERR_WORKSPACE before anything is launched.  The first call on a device
 * looks up the array's device address (cudaGetSymbolAddress) with that device
 * current; make that first call before any stream capture.  The call itself
 * allocates nothing.  All calls share the one array and nothing in it needs
 * to start at zero, but calls that overlap on the GPU (different streams, or
 * concurrent host threads) race on it: serialise them.
 */
int gdn2_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *log_alpha,
                           const void *b, const void *w, const float *S0, void *o, float *S_T,
                           int B, int T, int H, int dk, int dv, int dtype, cudaStream_t stream);

/*
 * Synchronises `stream`, then returns and clears the device status word of
 * the current device: GDN2_OK, GDN2_ERR_TIMEOUT (a bounded device wait ran
 * out) or GDN2_ERR_CUDA (the stream reported an error).
 */
int gdn2_get_device_status(cudaStream_t stream);

/* Static, human-readable name of a gdn2_status value. */
const char *gdn2_status_string(int status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int gdn2_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN2_H */
