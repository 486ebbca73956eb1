// Host-side construction of the TMA tensor maps the tcgen05 kernels load
// their tiles with.  cuTensorMapEncodeTiled is reached through the runtime's
// driver entry point, so the library does not link the driver library itself.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn2 {

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

// A [B, T, H, D] bf16 token tensor, read in boxes of 64 channels x 64 tokens
// of one head with the 128-byte swizzle: one box is a [64][64] block of the
// kernels' swizzled tiles.  Tokens past T read as zeros.
inline bool token_tensor_map(CUtensorMap *m, const void *base, int B, int T, int H, int D) {
    const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)T * H * D * 2};
    const cuuint32_t box[4] = {64, 1, 64, 1};
    const cuuint32_t unit[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, unit,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same tensor read as whole [64 tokens][128 channels] tiles in one box:
// a 5D view (64 channels, token, channel half, head, batch) whose box {64, 64,
// 2, 1, 1} lands as the kernels' tile layout, two [64][64] swizzled blocks
// (channel halves) one after the other.  The channel-half stride (128 bytes)
// lies below the token stride: the dimensions need not be ordered by stride.
inline bool token_tile_map(CUtensorMap *m, const void *base, int B, int T, int H, int D) {
    const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc || D != 128) return false;
    const cuuint64_t dims[5] = {64, (cuuint64_t)T, 2, (cuuint64_t)H, (cuuint64_t)B};
    const cuuint64_t strides[4] = {(cuuint64_t)H * D * 2, 128, (cuuint64_t)D * 2, (cuuint64_t)T * H * D * 2};
    const cuuint32_t box[5] = {64, 64, 2, 1, 1};
    const cuuint32_t unit[5] = {1, 1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void *>(base), dims, strides, box, unit,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace gdn2
