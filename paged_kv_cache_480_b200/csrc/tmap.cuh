// Host-side tensor-map encoding (TMA descriptors) through the driver's
// cuTensorMapEncodeTiled, looked up once through the runtime, so the
// library links no driver library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>

namespace pkv {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn tensor_map_encoder() {
    static std::atomic<EncodeTiledFn> cached{nullptr};
    EncodeTiledFn fn = cached.load(std::memory_order_acquire);
    if (fn) return fn;
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult found = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &found) != cudaSuccess ||
        found != cudaDriverEntryPointSuccess || ptr == nullptr)
        return nullptr;
    fn = reinterpret_cast<EncodeTiledFn>(ptr);
    cached.store(fn, std::memory_order_release);
    return fn;
}

// Tiled map over a row-major tensor (innermost dimension first), zero fill
// out of bounds.  Returns false if the driver rejects it.
inline bool encode_tiled(CUtensorMap* map, CUtensorMapDataType type, int rank, const void* base,
                         const cuuint64_t* dims, const cuuint64_t* strides_bytes, const cuuint32_t* box,
                         CUtensorMapSwizzle swizzle) {
    EncodeTiledFn fn = tensor_map_encoder();
    if (!fn) return false;
    const cuuint32_t elem_strides[5] = {1, 1, 1, 1, 1};
    return fn(map, type, (cuuint32_t)rank, const_cast<void*>(base), dims, strides_bytes, box, elem_strides,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace pkv
