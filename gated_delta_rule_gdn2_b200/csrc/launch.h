// Internal launcher interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace gdn2 {

// Token tensors [B, T, H, D]; the decode step uses T = 1 ([B, H, D]).
struct RecurrentArgs {
    const void *q, *k, *v, *log_alpha, *b, *w;
    const float *S_in;  // initial state or nullptr (zero)
    float *S_out;       // final state or nullptr
    void *o;
    int B, T, H;
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
};

// Bytes per chunk of the saved intra-chunk tiles (T, M: 64x64 bf16; U: 64 x dv bf16).
__host__ __device__ inline size_t intra_tile_bytes(int dv) { return (size_t)2 * 64 * 64 * 2 + (size_t)64 * dv * 2; }
// The saved-state buffer: the chunk-boundary states, then (256-byte aligned) the intra tiles.
inline size_t states_region_bytes(int B, int T, int H, int dk, int dv) {
    const size_t nc = (size_t)((T + 63) / 64);
    return ((size_t)B * H * (nc + 1) * dk * dv * 2 + 255) / 256 * 256;
}
inline size_t intra_region_bytes(int B, int T, int H, int dv) {
    const size_t nc = (size_t)((T + 63) / 64);
    return ((size_t)B * H * nc * intra_tile_bytes(dv) + 255) / 256 * 256;
}
// Then, for dk = dv = 128 (the tensor-memory kernels), the decayed operands
// Qt, Gt and Kb (or Kt) of every chunk, 3 x 64 x 128 bf16 each.
constexpr size_t kOpsTileBytes = (size_t)3 * 64 * 128 * 2;
inline size_t ops_region_bytes(int B, int T, int H, int dk, int dv) {
    if (dk != 128 || dv != 128) return 0;
    const size_t nc = (size_t)((T + 63) / 64);
    return (size_t)B * H * nc * kOpsTileBytes;
}

cudaError_t launch_chunk_bwd_tc(const ChunkBwdArgs &a, cudaStream_t s);  // reverse pass, dk = dv = 128, tcgen05
cudaError_t launch_chunk_bwd(const ChunkBwdArgs &a, int dk, int dv, cudaStream_t s);
size_t chunk_bwd_ws_bytes(int B, int T, int H, int dk, int dv, size_t *scr_stride, size_t *states_bytes);

cudaError_t launch_recurrent_fwd(const RecurrentArgs &a, int dk, int dv, bool bf16, cudaStream_t s);
cudaError_t launch_recurrent_bwd(const RecurrentBwdArgs &a, int dk, int dv, bool bf16, cudaStream_t s);
size_t recurrent_bwd_ws_bytes(int B, int T, int H, int dk, int dv);

}  // namespace gdn2
