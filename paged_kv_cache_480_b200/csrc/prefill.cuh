// Host-side launch of the paged prefill kernel.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "pagedkv.h"

namespace pkv {

struct PrefillArgs {
    void* out;
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    const int32_t* context_lens;
    const int32_t* query_start_loc;
    unsigned int* errors;
    float scale;
    int num_tokens, num_seqs, num_heads, num_kv_heads, head_size, block_size, num_blocks;
    int max_blocks_per_seq, max_query_len;
    pkv_dtype dtype;
    uint32_t wait_limit;   // polls before a bounded wait gives up
};

// Largest group (query heads per KV head) of the prefill kernel: one query
// tile of 128 rows holds 128 / G queries of G heads each.
constexpr int kPrefillMaxGroup = 128;

// Encodes the tensor maps and launches; PKV_ERR_UNSUPPORTED for shapes with
// no kernel, PKV_ERR_CUDA if the driver's tensor-map encoder or the launch fails.
pkv_status launch_prefill(const PrefillArgs& a, cudaStream_t stream);

}  // namespace pkv
