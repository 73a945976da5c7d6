// Host-side encoding of TMA tensor maps (cuTensorMapEncodeTiled, fetched from
// the driver at run time so the library does not link libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace moda {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    return fn;
}

// 4-D bf16 map with 128-byte swizzle; dims and byte strides innermost first.
// Out-of-range box elements of a load read as zero.
inline bool make_tmap_bf16_4d(CUtensorMap* m, const void* base, const cuuint64_t dims[4],
                              const cuuint64_t strides_b[3], const cuuint32_t box[4]) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    const cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides_b, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 4-D map of bytes (8-bit depth codes) without swizzle: rows land in shared
// memory as plain 128-byte lines for the in-place dequantisation.
inline bool make_tmap_u8_4d(CUtensorMap* m, const void* base, const cuuint64_t dims[4],
                            const cuuint64_t strides_b[3], const cuuint32_t box[4]) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    const cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides_b, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace moda
