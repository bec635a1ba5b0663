// Parameter blocks and launchers of the cache-maintenance kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace pkv {

struct CacheWriteParams {
    const unsigned char* key;
    const unsigned char* value;
    unsigned char* k_cache;
    unsigned char* v_cache;
    const int64_t* slot_mapping;
    unsigned int* errors;
    int64_t key_stride_bytes;    // between tokens
    int64_t value_stride_bytes;
    int64_t row_bytes;           // head_size * element size (multiple of 16)
    int num_tokens, num_kv_heads, block_size, num_blocks;
};

constexpr int kMaxLayers = 256;

struct CopyBlocksParams {
    void* k[kMaxLayers];
    void* v[kMaxLayers];
    const int64_t* block_mapping;   // [pairs][2]
    unsigned int* errors;
    int64_t block_bytes;
    int64_t num_blocks;
    int num_pairs;
};

struct SwapBlocksParams {
    const void* src[2 * kMaxLayers];
    void* dst[2 * kMaxLayers];
    const int64_t* block_mapping;   // [pairs][2] (src, dst), device-accessible
    unsigned int* errors;
    int64_t block_bytes;
    int64_t src_blocks, dst_blocks;
    int num_pairs;
};

struct CacheWriteFp8Params {
    const void* key;
    const void* value;
    unsigned char* k_cache;        // E4M3 bytes, [NB][Hkv][bs][D]
    unsigned char* v_cache;
    const int64_t* slot_mapping;
    unsigned int* errors;
    int64_t key_stride, value_stride;   // elements between tokens
    float k_scale, v_scale;
    int num_tokens, num_kv_heads, head_size, block_size, num_blocks;
    int src_dtype;                 // pkv_dtype of key / value
};

cudaError_t launch_reshape_and_cache_fp8(const CacheWriteFp8Params& p, int num_sms,
                                         cudaStream_t stream);

cudaError_t launch_swap_blocks(const SwapBlocksParams& p, int num_pairs, int num_caches,
                               cudaStream_t stream);

cudaError_t launch_reshape_and_cache(const CacheWriteParams& p, int num_sms, cudaStream_t stream);
cudaError_t launch_copy_blocks(const CopyBlocksParams& p, int num_pairs, int num_layers,
                               cudaStream_t stream);

}  // namespace pkv
