// Host-side dispatch of the decode and merge kernels over the supported
// (head_size, block_size, group size) combinations for one pair of element
// types: TQ for q and out, TC for the caches.
#pragma once

#include <atomic>

#include "decode_kernel.cuh"
#include "merge_kernel.cuh"

namespace pkv {

constexpr int kMaxDevices = 64;
constexpr int kMaxDynSmem = 232448 - 1024;  // 227 KB opt-in per CTA on sm_100, less static smem

template <typename TQ, typename TC, int D, int BS, int G>
cudaError_t run_decode(const DecodeParams& p, dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream) {
    static std::atomic<bool> configured[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    auto kernel = paged_decode_kernel<TQ, TC, D, BS, G>;
    if (dev >= 0 && dev < kMaxDevices && !configured[dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxDynSmem);
        if (e != cudaSuccess) return e;
        configured[dev].store(true, std::memory_order_release);
    }
    return launch_pdl(kernel, grid, block, smem, stream, p);
}

#define PKV_FOR_EACH_SHAPE(X) \
    X(64, 16, 1) X(64, 16, 2) X(64, 16, 4) X(64, 16, 8)     \
    X(64, 32, 1) X(64, 32, 2) X(64, 32, 4) X(64, 32, 8)     \
    X(128, 16, 1) X(128, 16, 2) X(128, 16, 4) X(128, 16, 8) \
    X(128, 32, 1) X(128, 32, 2) X(128, 32, 4) X(128, 32, 8)

template <typename TQ, typename TC>
cudaError_t dispatch_decode(const DecodeParams& p, int D, int BS, int G, dim3 grid, dim3 block,
                            size_t smem, cudaStream_t stream) {
#define PKV_CASE(d, bs, g) \
    if (D == d && BS == bs && G == g) return run_decode<TQ, TC, d, bs, g>(p, grid, block, smem, stream);
    PKV_FOR_EACH_SHAPE(PKV_CASE)
#undef PKV_CASE
    return cudaErrorInvalidValue;
}

// Bytes of one warp's shared-memory region for R stages (0 if unsupported).
template <typename TQ, typename TC>
uint32_t decode_warp_smem(int D, int BS, int G, int R) {
#define PKV_CASE(d, bs, g) \
    if (D == d && BS == bs && G == g) return WarpSmem<TQ, TC, d, bs, g>::bytes(R);
    PKV_FOR_EACH_SHAPE(PKV_CASE)
#undef PKV_CASE
    return 0;
}

template <typename T>
cudaError_t dispatch_merge(const ReduceParams& p, int D, cudaStream_t stream) {
    const size_t smem = sizeof(float2) * (size_t)p.max_parts;
    const dim3 grid(p.num_seqs, p.num_heads);
    if (D == 64) return launch_pdl(lse_merge_kernel<T, 64>, grid, dim3(128), smem, stream, p);
    if (D == 128) return launch_pdl(lse_merge_kernel<T, 128>, grid, dim3(128), smem, stream, p);
    return cudaErrorInvalidValue;
}

}  // namespace pkv

// One set of entry points per (q type, cache type), defined in decode_<name>.cu.
#define PKV_DECLARE_TYPES(name)                                                                  \
    namespace pkv {                                                                             \
    cudaError_t decode_##name(const DecodeParams& p, int D, int BS, int G, dim3 grid, dim3 block, \
                              size_t smem, cudaStream_t stream);                                \
    uint32_t warp_smem_##name(int D, int BS, int G, int R);                                     \
    }

#define PKV_DEFINE_TYPES(name, TQ, TC)                                                          \
    namespace pkv {                                                                             \
    cudaError_t decode_##name(const DecodeParams& p, int D, int BS, int G, dim3 grid, dim3 block, \
                              size_t smem, cudaStream_t stream) {                               \
        return dispatch_decode<TQ, TC>(p, D, BS, G, grid, block, smem, stream);                 \
    }                                                                                           \
    uint32_t warp_smem_##name(int D, int BS, int G, int R) {                                    \
        return decode_warp_smem<TQ, TC>(D, BS, G, R);                                           \
    }                                                                                           \
    }

#define PKV_DECLARE_MERGE(name)                                                                  \
    namespace pkv {                                                                             \
    cudaError_t merge_##name(const ReduceParams& p, int D, cudaStream_t stream);                \
    }

#define PKV_DEFINE_MERGE(name, T)                                                               \
    namespace pkv {                                                                             \
    cudaError_t merge_##name(const ReduceParams& p, int D, cudaStream_t stream) {               \
        return dispatch_merge<T>(p, D, stream);                                                 \
    }                                                                                           \
    }

PKV_DECLARE_TYPES(f32)
PKV_DECLARE_TYPES(f16)
PKV_DECLARE_TYPES(bf16)
PKV_DECLARE_TYPES(f32_fp8)
PKV_DECLARE_TYPES(f16_fp8)
PKV_DECLARE_TYPES(bf16_fp8)
PKV_DECLARE_MERGE(f32)
PKV_DECLARE_MERGE(f16)
PKV_DECLARE_MERGE(bf16)
