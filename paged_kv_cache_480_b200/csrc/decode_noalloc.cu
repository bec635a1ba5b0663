// paged_attention_decode_noalloc: the decode step for callers that cannot
// allocate device memory and have no buffer to lend as workspace.
//
// Some callers may not call cudaMalloc at all: a plug-in inside a host
// framework that owns every device allocation through its own arena, or a
// latency-critical loop that cannot afford cudaMalloc's implicit device
// synchronisation.  This entry point needs nothing from them but the inputs
// and the output: its scratch (work counters, partition prefix sums and
// split-context partials) is one fixed array in this file, reserved on every
// GPU that loads the library for as long as the process lives.
#include <atomic>

#include "pagedkv.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[PKV_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device.  In host code
// the array's name stands for a host-side shadow, so its address is looked up
// once per device with that device current.
pkv_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKV_ERR_CUDA;
    void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return PKV_ERR_CUDA;
        g_scratch_ptr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return PKV_OK;
}

}  // namespace

extern "C" pkv_status paged_attention_decode_noalloc(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, const int32_t* context_lens, float scale, int num_kv_heads,
    int block_size, int num_seqs, int num_heads, int head_size, int num_blocks,
    int max_blocks_per_seq, int max_context_len, pkv_dtype dtype, int partition_size,
    void* stream) {
    const size_t need = paged_attention_workspace_size(num_seqs, num_heads, num_kv_heads, head_size,
                                                       block_size, max_context_len, dtype,
                                                       partition_size);
    if (need == 0) {
        // Let the regular checks name the argument problem (nothing is launched).
        return paged_attention_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                                      num_kv_heads, block_size, num_seqs, num_heads, head_size,
                                      num_blocks, max_blocks_per_seq, max_context_len, dtype,
                                      partition_size, nullptr, 0, stream);
    }
    if (need > (size_t)PKV_NOALLOC_SCRATCH_BYTES) return PKV_ERR_WORKSPACE;
    void* scratch = nullptr;
    pkv_status st = scratch_address(&scratch);
    if (st != PKV_OK) return st;
    // The array keeps whatever the previous call left: zero the scheduling
    // counters, which must start at zero (the rest is written before read).
    if (cudaMemsetAsync(scratch, 0, 256, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return PKV_ERR_CUDA;
    return paged_attention_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                                  num_kv_heads, block_size, num_seqs, num_heads, head_size,
                                  num_blocks, max_blocks_per_seq, max_context_len, dtype,
                                  partition_size, scratch, PKV_NOALLOC_SCRATCH_BYTES, stream);
}
