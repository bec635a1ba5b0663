// Host-side launch of the tensor-core split-context decode (decode_tc_kernel.cuh)
// followed by its log-sum-exp merge.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "pagedkv.h"

namespace pkv {

// Smallest group (query heads per KV head) that takes the tensor-core decode
// for 16-bit q and caches.
#ifndef PKV_DECODE_TC_MIN_GROUP
#define PKV_DECODE_TC_MIN_GROUP 16
#endif
constexpr int kDecodeTcMinGroup = PKV_DECODE_TC_MIN_GROUP;

struct DecodeTcArgs {
    void* out;
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    const int32_t* context_lens;
    unsigned int* errors;
    int32_t* prefix;     // [S + 1] workspace
    float* part_acc;     // [decode_tc_partial_rows(...)][D]
    float2* part_ml;     // [decode_tc_partial_rows(...)]
    float scale;
    int num_seqs, num_heads, num_kv_heads, head_size, block_size, num_blocks;
    int max_blocks_per_seq, max_context_len;
    pkv_dtype dtype;
    uint32_t wait_limit;
};

// Partial-result rows of the tensor-core decode: every CTA writes, for each
// of the units its tile range touches and for each of its two halves, one
// slot of min(G, 128) rows at 2 * (cta + unit) + half; units = sequences x
// KV heads x ceil(G / 128) slices.
size_t decode_tc_partial_rows(int num_seqs, int num_heads, int num_kv_heads);

// Encodes the tensor maps, launches the decode and the merge.
pkv_status launch_decode_tc(const DecodeTcArgs& a, cudaStream_t stream);

}  // namespace pkv
