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
 * - The library keeps, per device, the device addresses of its own device
 *   variables (the status word, the no-alloc scratch) from its first call on
 *   that device.  A device or primary-context reset (cudaDeviceReset) makes
 *   them stale: do not reset a device while this library is in use on it.
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
 * For bf16 with too few sequences to fill the GPU this is the size of the
 * sequence-segmented forward (below): dk = dv = 128 with T a multiple of 64,
 * at least 16 chunks and B*H*3 <= the SM count; dk = dv = 64 with T a
 * multiple of 4 segments of at least 8 chunks and B*H*4 <= the SM count.
 * Otherwise, and always for fp32, it is the one-CTA-per-sequence forward's
 * B*H*64*dk*4 bytes.
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
 * segmented one, each sequence runs as P segments side by side: the state
 * update of a chunk is affine in the state (Gated Delta Rule-2 section of
 * "Why NVIDIA Gated DeltaNet-2 separates erase and write gates").  For
 * dk = dv = 128 the segments are runs of whole chunks; one launch runs every
 * segment from zero (the first from S0) and, beside it, the transition of
 * every later segment (from I with no write term, together with the rows
 * Phi_t^T q_t); an fp32 scan gives the segments' start states and S_T, and a
 * tensor-core pass adds S_start^T Phi_t^T q_t to o (about two forwards of work
 * on up to 2P - 1 times as many SMs).  For dk = dv = 64 two forwards give
 * every segment's local end state and transition, the scan the start states,
 * and a third forward o and S_T.  Same results to bf16 rounding.
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
 * Few long sequences (bf16, dk = dv = 128, where gdn2_chunk_fwd_workspace
 * gives the segmented size): the pair splits every sequence into P segments
 * (segmented training).  The forward finds each segment's start state with
 * the segmented forward and then keeps the states and tiles of the segments
 * as a packed batch; the backward runs over the segments twice, first from
 * zero end gradients (each segment's own start-state gradient), then from the
 * end gradients a reverse scan through the segments' transitions gives.  The
 * choice follows from B, T, H, dk, dv alone, and the sizes
 * (gdn2_chunk_states_bytes, gdn2_chunk_fwd_workspace,
 * gdn2_chunk_bwd_saved_workspace) are those of that path; the forward then
 * needs the full gdn2_chunk_fwd_workspace (GDN2_ERR_WORKSPACE otherwise).
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
 * Packed variable-length batches (documents of different lengths in one
 * call, with no padding).  The token tensors are [total_T, H, D] (the rows of
 * all N sequences back to back; equivalently [1, total_T, H, D]); sequence n
 * is rows cu_seqlens[n] .. cu_seqlens[n+1] - 1.  cu_seqlens: DEVICE int32
 * array of N + 1 nondecreasing offsets, cu_seqlens[0] = 0, cu_seqlens[N] =
 * total_T, 4-byte aligned; a sequence may be empty.  States (S0, S_T, dS_T,
 * dS0) are [N, H, dk, dv] fp32, one per sequence.  Each sequence evolves
 * from its own S0 exactly as a gdn2_chunk_fwd call on it alone would (the
 * "1.3B params & 100B tokens" section of "Why NVIDIA Gated DeltaNet-2
 * separates erase and write gates" trains on packed 4K-token documents; the
 * state does not carry across a document boundary).  The offsets are read on
 * the device only: a sequence whose offsets are out of range (negative,
 * decreasing, or past total_T) is skipped and GDN2_ERR_INVALID_ARG is
 * recorded in the device status word (gdn2_get_device_status).
 * Arguments otherwise as the fixed-length calls, with (N, total_T) in place
 * of (B, T).  Packed batches always run one CTA per sequence (never the
 * sequence-segmented forward).  The saved-state pair keeps its buffer in a
 * private layout sized by gdn2_chunk_states_varlen_bytes(N, total_T, ...),
 * which depends only on N and total_T, not on the individual lengths.
 */
size_t gdn2_chunk_fwd_varlen_workspace(int N, int total_T, int H, int dk, int dv, int dtype);
int gdn2_chunk_fwd_varlen(const void *q, const void *k, const void *v, const void *log_alpha,
                          const void *b, const void *w, const float *S0, void *o, float *S_T,
                          const int *cu_seqlens, int N, int total_T, int H, int dk, int dv, int dtype,
                          void *ws, size_t ws_bytes, cudaStream_t stream);
size_t gdn2_chunk_bwd_varlen_workspace(int N, int total_T, int H, int dk, int dv, int dtype);
int gdn2_chunk_bwd_varlen(const void *q, const void *k, const void *v, const void *log_alpha,
                          const void *b, const void *w, const float *S0, const void *dO,
                          const float *dS_T, void *dq, void *dk_, void *dv_, void *dlog_alpha,
                          void *db, void *dw, float *dS0, const int *cu_seqlens,
                          int N, int total_T, int H, int dk, int dv, int dtype,
                          void *ws, size_t ws_bytes, cudaStream_t stream);
size_t gdn2_chunk_states_varlen_bytes(int N, int total_T, int H, int dk, int dv, int dtype);
int gdn2_chunk_fwd_save_varlen(const void *q, const void *k, const void *v, const void *log_alpha,
                               const void *b, const void *w, const float *S0, void *o, float *S_T,
                               void *states, const int *cu_seqlens, int N, int total_T, int H, int dk,
                               int dv, int dtype, void *ws, size_t ws_bytes, cudaStream_t stream);
size_t gdn2_chunk_bwd_saved_varlen_workspace(int N, int total_T, int H, int dk, int dv, int dtype);
int gdn2_chunk_bwd_saved_varlen(const void *q, const void *k, const void *v, const void *log_alpha,
                                const void *b, const void *w, const float *S0, const void *dO,
                                const float *dS_T, const void *states, void *dq, void *dk_, void *dv_,
                                void *dlog_alpha, void *db, void *dw, float *dS0,
                                const int *cu_seqlens, int N, int total_T, int H, int dk, int dv,
                                int dtype, void *ws, size_t ws_bytes, cudaStream_t stream);

/*
 * Reduced gates ("GDN-2 in one minute" on the orcarouter GDN-2-3B page, and
 * the Gated Delta Rule-2 section of the axbrief page: GDN-2 with b = w = beta
 * is KDA's update S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} +
 * beta_t k_t v_t^T, and with a scalar alpha_t as well it is Gated DeltaNet's).
 * `beta` is one scalar per token and head, [B, T, H] (decode: [B, H]), in
 * the token dtype, and stands for both the erase gate b = beta 1 and the
 * write gate w = beta 1.  The *_kda calls take log_alpha per key channel
 * ([B, T, H, dk]); the *_gdn calls take a scalar decay log_alpha [B, T, H]
 * (decode: [B, H]).  Results are those of the general call with the gates
 * expanded to vectors (the forward's bit for bit); the chunk kernels fill the
 * gate tiles from the scalars on chip instead of reading expanded tensors.
 * The backward returns dbeta [B, T, H] = sum_c db[c] + sum_j dw[j] and, for
 * GDN, dlog_alpha [B, T, H] = sum_c dlog_alpha[c] (dq, dk_, dv_ and, for KDA,
 * dlog_alpha as in gdn2_chunk_bwd).  Workspaces: gdn2_chunk_fwd_workspace /
 * gdn2_chunk_bwd_workspace.  Supported: decode for every size and dtype; the
 * chunk forward for bf16 with dk = dv = 128 and for fp32; the chunk backward
 * for bf16 with dk = dv = 128.  Other combinations: GDN2_ERR_UNSUPPORTED.
 * A scalar-gate tensor needs only element alignment.
 */
int gdn2_chunk_fwd_kda(const void *q, const void *k, const void *v, const void *log_alpha,
                       const void *beta, const float *S0, void *o, float *S_T,
                       int B, int T, int H, int dk, int dv, int dtype,
                       void *ws, size_t ws_bytes, cudaStream_t stream);
int gdn2_chunk_fwd_gdn(const void *q, const void *k, const void *v, const void *log_alpha,
                       const void *beta, const float *S0, void *o, float *S_T,
                       int B, int T, int H, int dk, int dv, int dtype,
                       void *ws, size_t ws_bytes, cudaStream_t stream);
int gdn2_chunk_bwd_kda(const void *q, const void *k, const void *v, const void *log_alpha,
                       const void *beta, const float *S0, const void *dO, const float *dS_T,
                       void *dq, void *dk_, void *dv_, void *dlog_alpha, void *dbeta, float *dS0,
                       int B, int T, int H, int dk, int dv, int dtype,
                       void *ws, size_t ws_bytes, cudaStream_t stream);
int gdn2_chunk_bwd_gdn(const void *q, const void *k, const void *v, const void *log_alpha,
                       const void *beta, const float *S0, const void *dO, const float *dS_T,
                       void *dq, void *dk_, void *dv_, void *dlog_alpha, void *dbeta, float *dS0,
                       int B, int T, int H, int dk, int dv, int dtype,
                       void *ws, size_t ws_bytes, cudaStream_t stream);
int gdn2_decode_step_kda(const void *q, const void *k, const void *v, const void *log_alpha,
                         const void *beta, float *S, void *o,
                         int B, int H, int dk, int dv, int dtype, cudaStream_t stream);
int gdn2_decode_step_gdn(const void *q, const void *k, const void *v, const void *log_alpha,
                         const void *beta, float *S, void *o,
                         int B, int H, int dk, int dv, int dtype, cudaStream_t stream);

/*
 * Layer prologue and epilogue ("Why NVIDIA Gated DeltaNet-2 separates erase
 * and write gates", section on implications for practitioners: the query and
 * key paths are a projection, a short causal convolution, SiLU and L2
 * normalisation; the value path a projection, a short convolution and SiLU;
 * the output an RMS normalisation with a SiLU output gate).  The projections
 * are matrix products outside this library; these calls take their outputs.
 *
 * gdn2_prologue_fwd: from the projected xq, xk [rows, H, dk], xv [rows, H,
 * dv] and the gate pre-activations xa, xb [rows, H, dk], xw [rows, H, dv],
 * one fused pass writes the mixer's inputs
 *   q = l2norm(silu(conv(xq, Wq))), k = l2norm(silu(conv(xk, Wk))),
 *   v = silu(conv(xv, Wv)), log_alpha = log sigmoid(xa), b = sigmoid(xb),
 *   w = sigmoid(xw)
 * in the same dtype.  conv is depthwise and causal: y[t, c] = sum_{j<K}
 * W[c][j] x[t - (K-1) + j, c] with W fp32 [H*D][K], K in 1..4, and taps
 * before a sequence's first token reading zero; l2norm(s) = s / sqrt(|s|^2 +
 * 1e-6) over the head dimension.  Sequences: a fixed-length batch
 * (cu_seqlens == NULL) is B sequences of T tokens ([B, T, H, D], rows = B*T);
 * a packed batch (cu_seqlens: B + 1 device int32 offsets, as for the _varlen
 * calls) is B sequences in T rows.  gdn2_prologue_bwd: the gradients of the
 * pre-activations and of the three filters (fp32 [H*D][K], summed over every
 * token in a fixed order: deterministic) from those of the mixer's inputs;
 * workspace gdn2_prologue_bwd_workspace(B, T, H, dk, dv, K, packed).
 *
 * gdn2_output_gate_fwd: z = o / sqrt(mean_j o_j^2 + 1e-6) * gamma * silu(g)
 * per token and head, o, g, z [rows, H, dv] in the token dtype, gamma fp32
 * [dv] shared by the heads.  gdn2_output_gate_bwd: do, dg and dgamma (fp32
 * [dv], deterministic sum) from dz; workspace
 * gdn2_output_gate_bwd_workspace(rows, H, dv).
 * Every pointer 16-byte aligned; dk, dv in {64, 128}; dtype GDN2_BF16 or
 * GDN2_FP32.  (The page gives no convolution width, norm epsilon or weight
 * shape: K is the caller's, 1e-6 and a head-shared gamma are this library's
 * reading.)
 */
int gdn2_prologue_fwd(const void *xq, const void *xk, const void *xv, const float *Wq,
                      const float *Wk, const float *Wv, int K, const void *xa, const void *xb,
                      const void *xw, void *q, void *k, void *v, void *log_alpha, void *b, void *w,
                      const int *cu_seqlens, int B, int T, int H, int dk, int dv, int dtype,
                      cudaStream_t stream);
size_t gdn2_prologue_bwd_workspace(int B, int T, int H, int dk, int dv, int K, int packed);
int gdn2_prologue_bwd(const void *xq, const void *xk, const void *xv, const float *Wq,
                      const float *Wk, const float *Wv, int K, const void *xa, const void *xb,
                      const void *xw, const void *dq, const void *dk_, const void *dv_,
                      const void *dlog_alpha, const void *db, const void *dw, void *dxq, void *dxk,
                      void *dxv, float *dWq, float *dWk, float *dWv, void *dxa, void *dxb, void *dxw,
                      const int *cu_seqlens, int B, int T, int H, int dk, int dv, int dtype,
                      void *ws, size_t ws_bytes, cudaStream_t stream);
/*
 * gdn2_chunk_fwd followed by the output epilogue, z = o / rms(o) * gamma *
 * silu(g) [B,T,H,dv] (o itself is not written).  For bf16 with dk = dv = 128
 * on the one-CTA-per-sequence path the epilogue runs inside the forward's
 * O epilogue, so o never goes to memory (the output-gate tile arrives by TMA
 * while the chunk's state update runs); otherwise the forward writes o into
 * z and gdn2_output_gate_fwd runs on it in place.  Arguments otherwise as
 * gdn2_chunk_fwd; g like o, gamma fp32 [dv].
 */
int gdn2_chunk_fwd_gated(const void *q, const void *k, const void *v, const void *log_alpha,
                         const void *b, const void *w, const float *S0, const void *g,
                         const float *gamma, void *z, float *S_T, int B, int T, int H, int dk, int dv,
                         int dtype, void *ws, size_t ws_bytes, cudaStream_t stream);
int gdn2_output_gate_fwd(const void *o, const void *g, const float *gamma, void *z,
                         long long rows, int H, int dv, int dtype, cudaStream_t stream);
size_t gdn2_output_gate_bwd_workspace(long long rows, int H, int dv);
int gdn2_output_gate_bwd(const void *o, const void *g, const float *gamma, const void *dz,
                         void *dO, void *dg, float *dgamma, long long rows, int H, int dv, int dtype,
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
 * GDN2_ERR_WORKSPACE before anything is launched.  The call passes the whole
 * array as gdn2_chunk_fwd's workspace, so it takes the sequence-segmented
 * path wherever gdn2_chunk_fwd_workspace(...) asks for that path's size and
 * the size fits in the array (e.g. B = 1, H = 1, T = 4096, dk = dv = 128),
 * and the one-CTA-per-sequence path otherwise; results equal gdn2_chunk_fwd's
 * with that workspace bit for bit.  The first call on a device
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

/*
 * Test knobs (no counterpart on the pages): they exist so that a test can
 * make a device-side bounded wait run out and check that the kernel gives
 * up cleanly, records GDN2_ERR_TIMEOUT and leaves the context usable.
 *   GDN2_DEBUG_WAIT_LIMIT: iterations of every bounded mbarrier wait of the
 *     chunk kernels launched from now on (0 = the default, a few seconds).
 *   GDN2_DEBUG_WITHHOLD_READY: the chunk index at which the bf16
 *     dk = dv = 128 forward withholds the arrival that hands a chunk's
 *     intra-chunk results to its state chain (-1 = none, the default); the
 *     chain's wait for it then runs out.  No copy or tensor-core operation
 *     depends on that arrival, so the kernel ends with none of them in flight.
 * Host-global settings of the process, not for production use; returns
 * GDN2_OK or GDN2_ERR_INVALID_ARG.
 */
enum { GDN2_DEBUG_WAIT_LIMIT = 0, GDN2_DEBUG_WITHHOLD_READY = 1 };
int gdn2_debug_set(int knob, long long value);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int gdn2_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN2_H */
