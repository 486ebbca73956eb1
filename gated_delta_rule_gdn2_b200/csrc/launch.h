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

// Chunk-parallel tensor-core forward (bf16 tokens).  ws: B*H*64*dk floats,
// used only by chunks whose in-chunk decay exceeds the fast path's range.
struct ChunkFwdArgs {
    const void *q, *k, *v, *log_alpha, *b, *w;
    const float *S0;
    void *o;
    float *S_T;
    float *ws;
    int B, T, H;
};

cudaError_t launch_chunk_fwd(const ChunkFwdArgs &a, int dk, int dv, cudaStream_t s);
size_t chunk_fwd_ws_bytes(int B, int H, int dk);

cudaError_t launch_recurrent_fwd(const RecurrentArgs &a, int dk, int dv, bool bf16, cudaStream_t s);
cudaError_t launch_recurrent_bwd(const RecurrentBwdArgs &a, int dk, int dv, bool bf16, cudaStream_t s);
size_t recurrent_bwd_ws_bytes(int B, int T, int H, int dk, int dv);

}  // namespace gdn2
