// Internal launcher interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gdn2 {

// Gate forms.  kGatesFull: b [.., dk] and w [.., dv] per token, log_alpha
// [.., dk].  kGatesKDA: one scalar beta per token and head stands for both
// gates (b = beta 1, w = beta 1; the args' b and w both point to beta
// [.., H]).  kGatesGDN: that, and a scalar decay (log_alpha [.., H]).
constexpr int kGatesFull = 0, kGatesKDA = 1, kGatesGDN = 2;

// Token tensors [B, T, H, D]; the decode step uses T = 1 ([B, H, D]).
struct RecurrentArgs {
    const void *q, *k, *v, *log_alpha, *b, *w;
    const float *S_in;  // initial state or nullptr (zero)
    float *S_out;       // final state or nullptr
    void *o;
    int B, T, H;
    const int *cu_seqlens = nullptr;  // packed variable-length sequences (see SeqView)
    int gates = kGatesFull;
};

struct RecurrentBwdArgs {
    const void *q, *k, *v, *log_alpha, *b, *w;
    const float *S0;
    const void *dO;
    const float *dS_T;
    void *dq, *dk, *dv, *dlog_alpha, *db, *dw;
    float *dS0;
    float *ws;
    int B, T, H;
    const int *cu_seqlens = nullptr;
    int gates = kGatesFull;
};

// Chunk-parallel tensor-core forward (bf16 tokens).  ws: per-CTA fp32
// scratch of ws_stride floats (>= 64*dk), used by chunks whose in-chunk decay
// exceeds the fast path's range.  states: optional bf16 [B*H][nchunks+1][dk][dv]
// output of the state at every chunk boundary (the backward's state pass);
// o may then be null.
struct ChunkFwdArgs {
    const void *q, *k, *v, *log_alpha, *b, *w;
    const float *S0;
    void *o;
    float *S_T;
    float *ws;
    size_t ws_stride;
    void *states;
    void *intra;  // optional: per chunk the bf16 tiles T, M (64x64 each) and U (64 x dv), as in shared memory
    void *ops;    // optional (dk = dv = 128): per chunk the bf16 operands Qt, Gt, Kb/Kt, as in shared memory
    int *status;  // device status word (bounded waits record GDN2_ERR_TIMEOUT here)
    int B, T, H;
    const int *cu_seqlens = nullptr;  // packed variable-length sequences (see SeqView)
    int gates = kGatesFull;           // gate form (kGatesKDA / kGatesGDN: dk = dv = 128 only)
    // test knobs (gdn2_debug_set): the bounded waits' iteration limit (0 = the
    // default) and a chunk whose intra-chunk hand-over arrival is withheld (-1 = none)
    uint32_t wait_limit = 0;
    int withhold_ready = -1;
    // output epilogue fused into the O epilogue (dk = dv = 128, no states kept):
    // o receives z = o / rms(o) * gamma * silu(out_gate), out_gate like o, gamma fp32 [dv]
    const void *out_gate = nullptr;
    const float *gamma = nullptr;
    // sequence segments (segments.cu, dk = dv = 128, fixed length, T a multiple
    // of 64): each sequence is cut into seg_P runs of whole chunks, and the
    // launch has B*H*(2 seg_P - 1) CTAs: first the local pass of every segment
    // (segment 0 from S0, the others from zero; o written in place; the end
    // state to seg_loc[(b*P + p)*H + h]), then the transition pass of segments
    // p = 1..P-1 (start I, no write term: v and w are not read; the rows
    // Phi_t^T q_t to seg_qphi, laid out like o; the transition to
    // seg_phi[(b*(P-1) + p-1)*H + h])
    int seg_P = 0;
    float *seg_loc = nullptr, *seg_phi = nullptr;
    void *seg_qphi = nullptr;
    // the warp-level kernel's transition pass (segments.cu, dk = dv): the state
    // starts from the identity and there is no write term (v and w are not read)
    bool transition = false;
};

cudaError_t launch_chunk_fwd(const ChunkFwdArgs &a, int dk, int dv, cudaStream_t s);
cudaError_t launch_chunk_fwd_tc(const ChunkFwdArgs &a, cudaStream_t s);  // dk = dv = 128, tcgen05
size_t chunk_fwd_ws_bytes(int B, int H, int dk);

// The plain forward for few long sequences as P sequence segments side by
// side (segments.cu): segment_count gives P (1 = not worth it), the
// workspace it needs, and the launch (S_T, o, status as in ChunkFwdArgs; the
// args' ws is ignored, `ws` of segments_ws_bytes holds everything).
int segment_count(int B, int T, int H, int dk, int dv);
size_t segments_ws_bytes(int B, int T, int H, int dk, int dv, int P);
cudaError_t launch_chunk_fwd_segments(const ChunkFwdArgs &a, int dk, int dv, int P, void *ws, cudaStream_t s);

// Segmented training (segments.cu): the saved-state pair for few long
// sequences at dk = dv = 128 (P = seg_train_count(...) > 1), with its own
// saved-buffer layout and workspaces.
struct ChunkBwdArgs;
int seg_train_count(int B, int T, int H, int dk, int dv);
size_t seg_train_states_bytes(int B, int T, int H, int P);
size_t seg_train_fwd_ws_bytes(int B, int T, int H, int P);
size_t seg_train_bwd_ws_bytes(int B, int T, int H, int P);
cudaError_t launch_seg_train_fwd(const ChunkFwdArgs &a, void *states, int P, void *ws, cudaStream_t s);
cudaError_t launch_seg_train_bwd(const ChunkBwdArgs &a, const void *states, int P, void *ws, cudaStream_t s);

// Chunk-parallel gate-aware backward (bf16 tokens): a state pass (the
// forward writing bf16 chunk-boundary states to `states`) and a reverse chunk
// pass.  scratch: per-CTA fp32 work area of scr_stride floats.
struct ChunkBwdArgs {
    const void *q, *k, *v, *log_alpha, *b, *w;
    const float *S0;
    const void *dO;
    const float *dS_T;
    void *dq, *dk, *dv, *dlog_alpha, *db, *dw;
    float *dS0;
    void *states;      // bf16 chunk-boundary states [B*H][nchunks+1][dk][dv]
    void *intra;       // per chunk the bf16 tiles T, M, U of the forward (intra_tile_bytes each)
    void *ops;         // dk = dv = 128: per chunk the forward's Qt, Gt, Kb/Kt (ops_tile_bytes each)
    float *scratch;
    size_t scr_stride;
    int *status;
    int states_given;  // 1: `states` already holds what the training forward kept
    int B, T, H;
    const int *cu_seqlens = nullptr;  // packed variable-length sequences (see SeqView)
    int gates = kGatesFull;           // gate form; KDA: db is dbeta [.., H] and dw unused; GDN: also dlog_alpha [.., H]
    uint32_t wait_limit = 0;          // test knob: the bounded waits' iteration limit (0 = the default)
};

// Bytes per chunk of the saved intra-chunk tiles (T, M: 64x64 bf16; U: 64 x dv bf16).
__host__ __device__ inline size_t intra_tile_bytes(int dv) { return (size_t)2 * 64 * 64 * 2 + (size_t)64 * dv * 2; }

// Where the tokens of sequence b lie, and where its per-chunk saved tiles and
// chunk-boundary states go.  A fixed-length batch (cu == nullptr) holds B
// sequences of T tokens, [B, T, H, D]; a packed variable-length batch holds B
// sequences in T token rows in all, [T, H, D], sequence b in rows
// cu[b] .. cu[b+1] - 1 (cu: B + 1 nondecreasing device int32, cu[0] = 0,
// cu[B] = T).  The saved buffers of a packed batch keep, per head, one slot
// per chunk from slot floor(cu[b] / 64) + b on (states: floor(cu[b] / 64) +
// 2 b on): consecutive sequences never overlap, since sequence b needs at most
// floor(cu[b+1] / 64) - floor(cu[b] / 64) + 1 chunk slots, and the slots of a
// head number at most floor(T / 64) + B (states: + 2 B).
__host__ __device__ inline size_t varlen_chunk_slots(int B, int T) { return (size_t)(T / 64) + (size_t)B; }
__host__ __device__ inline size_t varlen_state_slots(int B, int T) { return (size_t)(T / 64) + 2 * (size_t)B; }
struct SeqView {
    size_t row0;   // first token row of the sequence
    int len;       // its tokens
    int nchunks;   // ceil(len / 64)
    size_t cslot;  // saved-tile slot of its chunk 0 (chunk n: cslot + n)
    size_t sslot;  // chunk-boundary state slot of its state 0 (state n: sslot + n)
    int map_b, map_t0;  // TMA coordinates (batch, token) of its first row
    bool ok;       // false: cu_seqlens out of range for this sequence
};
__device__ __forceinline__ SeqView seq_view(const int *cu, int b, int h, int B, int T, int H) {
    SeqView v;
    if (!cu) {
        v.row0 = (size_t)b * T;
        v.len = T;
        v.nchunks = (T + 63) / 64;
        v.cslot = ((size_t)b * H + h) * v.nchunks;
        v.sslot = ((size_t)b * H + h) * (v.nchunks + 1);
        v.map_b = b;
        v.map_t0 = 0;
        v.ok = true;
        return v;
    }
    const int r0 = cu[b], r1 = cu[b + 1];
    v.ok = r0 >= 0 && r0 <= r1 && r1 <= T;
    if (!v.ok) {
        v.row0 = 0; v.len = 0; v.nchunks = 0; v.cslot = 0; v.sslot = 0; v.map_b = 0; v.map_t0 = 0;
        return v;
    }
    v.row0 = (size_t)r0;
    v.len = r1 - r0;
    v.nchunks = (v.len + 63) / 64;
    v.cslot = (size_t)h * varlen_chunk_slots(B, T) + (size_t)(r0 / 64) + b;
    v.sslot = (size_t)h * varlen_state_slots(B, T) + (size_t)(r0 / 64) + 2 * (size_t)b;
    v.map_b = 0;
    v.map_t0 = r0;
    return v;
}

// The saved-state buffer: the chunk-boundary states, then (256-byte aligned) the intra tiles.
__host__ __device__ inline size_t chunk_slots(int B, int T, int H, bool varlen) {
    return varlen ? (size_t)H * varlen_chunk_slots(B, T) : (size_t)B * H * (size_t)((T + 63) / 64);
}
__host__ __device__ inline size_t state_slots(int B, int T, int H, bool varlen) {
    return varlen ? (size_t)H * varlen_state_slots(B, T) : (size_t)B * H * (size_t)((T + 63) / 64 + 1);
}
inline size_t states_region_bytes(int B, int T, int H, int dk, int dv, bool varlen = false) {
    return (state_slots(B, T, H, varlen) * dk * dv * 2 + 255) / 256 * 256;
}
inline size_t intra_region_bytes(int B, int T, int H, int dv, bool varlen = false) {
    return (chunk_slots(B, T, H, varlen) * intra_tile_bytes(dv) + 255) / 256 * 256;
}
// Then, for dk = dv = 128 (the tensor-memory kernels), the decayed operands
// Qt, Gt and Kb (or Kt) of every chunk, 3 x 64 x 128 bf16 each.
constexpr size_t kOpsTileBytes = (size_t)3 * 64 * 128 * 2;
inline size_t ops_region_bytes(int B, int T, int H, int dk, int dv, bool varlen = false) {
    if (dk != 128 || dv != 128) return 0;
    return chunk_slots(B, T, H, varlen) * kOpsTileBytes;
}

cudaError_t launch_chunk_bwd_tc(const ChunkBwdArgs &a, cudaStream_t s);  // reverse pass, dk = dv = 128, tcgen05
cudaError_t launch_chunk_bwd(const ChunkBwdArgs &a, int dk, int dv, cudaStream_t s);
size_t chunk_bwd_ws_bytes(int B, int T, int H, int dk, int dv, size_t *scr_stride, size_t *states_bytes,
                          bool varlen = false);

cudaError_t launch_recurrent_fwd(const RecurrentArgs &a, int dk, int dv, bool bf16, cudaStream_t s);
cudaError_t launch_recurrent_bwd(const RecurrentBwdArgs &a, int dk, int dv, bool bf16, cudaStream_t s);
size_t recurrent_bwd_ws_bytes(int B, int T, int H, int dk, int dv, bool varlen = false);

}  // namespace gdn2
