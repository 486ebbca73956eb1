// gdn2_chunk_fwd_noalloc: the chunk-parallel forward for callers that cannot
// allocate device memory.
//
// Some callers run where cudaMalloc is unavailable or forbidden: inside a
// pre-sized memory pool they do not own, in an embedding runtime that hands
// out no device allocations, or on a code path that must not allocate (for
// instance one that runs while the caller's allocator is locked).  They can
// still pass their input and output buffers, but not the forward's scratch
// workspace.  This entry point supplies that scratch from a fixed array in
// the library's own device image instead.
//
// The array below is a file-scope __device__ object: every GPU that loads the
// library holds it (kScratchBytes) until the process exits.  In host code its
// name is only a host-side stand-in, so the device address is looked up with
// cudaGetSymbolAddress once per device (on the first call made with that
// device current) and passed to the kernels as an ordinary pointer.
#include "gdn2.h"

#include <cuda_runtime.h>

namespace {

// 8 MiB: B*H*dk <= 32768 (e.g. B*H <= 256 sequences at dk = 128).
constexpr size_t kScratchBytes = size_t(8) << 20;
__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void *g_scratch_ptr[kMaxDevices] = {nullptr};

}  // namespace

extern "C" int gdn2_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *log_alpha,
                                      const void *b, const void *w, const float *S0, void *o, float *S_T,
                                      int B, int T, int H, int dk, int dv, int dtype, cudaStream_t stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return GDN2_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return GDN2_ERR_UNSUPPORTED;
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
            (void)cudaGetLastError();
            return GDN2_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    // The ordinary entry point does all argument checks; a problem whose
    // workspace exceeds kScratchBytes gets GDN2_ERR_WORKSPACE before any launch.
    return gdn2_chunk_fwd(q, k, v, log_alpha, b, w, S0, o, S_T, B, T, H, dk, dv, dtype, g_scratch_ptr[dev],
                          kScratchBytes, stream);
}
