// Cache maintenance kernels: the cache write (each new token's K/V into its
// slot) and the copy-on-write block copy.  Both are bit copies of 16-byte
// chunks; neither converts data.
//
// reshape_and_cache: "PyTorch-CUDA-v2.9 image enables PagedAttention",
//   PagedAttention section (each decode step appends the new token's
//   key/value) and workflow list (prefill writes the tokens' KV into pages).
// copy_blocks: "Efficient Memory Management for Large Language Model Serving
//   with PagedAttention" summary page, sections 1 and 2 (reference counts and
//   copy-on-write for parallel sampling and shared prefixes).
#include "cache_ops.cuh"
#include "common.cuh"

namespace pkv {

// One thread per 16-byte chunk of one (token, KV head) row of K and of V.
__global__ void reshape_and_cache_kernel(const CacheWriteParams p) {
    griddep_wait();
    griddep_launch();
    const int64_t chunks_per_row = p.row_bytes / 16;
    const int64_t per_token = (int64_t)p.num_kv_heads * chunks_per_row;
    const int64_t total = (int64_t)p.num_tokens * per_token;
    const int64_t pool_slots = (int64_t)p.num_blocks * p.block_size;
    for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < total;
         w += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = w / per_token;
        const int64_t rem = w - i * per_token;
        const int64_t g = rem / chunks_per_row;
        const int64_t ch = rem - g * chunks_per_row;
        const int64_t slot = p.slot_mapping[i];
        if (slot < 0) continue;
        if (slot >= pool_slots) {
            if (rem == 0) flag_error(p.errors, PKV_DEVERR_SLOT);
            continue;
        }
        const int64_t blk = slot / p.block_size, off = slot - blk * p.block_size;
        const int64_t dst = ((blk * p.num_kv_heads + g) * p.block_size + off) * p.row_bytes + ch * 16;
        const uint4 kv = *reinterpret_cast<const uint4*>(p.key + i * p.key_stride_bytes +
                                                         g * p.row_bytes + ch * 16);
        const uint4 vv = *reinterpret_cast<const uint4*>(p.value + i * p.value_stride_bytes +
                                                         g * p.row_bytes + ch * 16);
        *reinterpret_cast<uint4*>(p.k_cache + dst) = kv;
        *reinterpret_cast<uint4*>(p.v_cache + dst) = vv;
    }
}

// Pairs are copied in parallel, so a pair whose destination is also another
// pair's destination or (within one pool) another pair's source, or whose
// source is another pair's destination, would make the result depend on the
// order the copies happen to run in.  Every CTA of a pair scans the whole
// mapping (all threads of the CTA take part); such a pair is skipped.
__device__ __forceinline__ bool pair_conflicts(const int64_t* map, int num_pairs, int pair, int64_t src,
                                               int64_t dst, bool same_pool) {
    bool hit = false;
    for (int j = threadIdx.x; j < num_pairs; j += blockDim.x) {
        if (j == pair) continue;
        const int64_t sj = map[2 * (int64_t)j], dj = map[2 * (int64_t)j + 1];
        hit |= dj == dst || (same_pool && (sj == dst || dj == src));
    }
    return __syncthreads_or(hit) != 0;
}

// grid = (pairs, layers, 2 caches); each CTA copies one block with 16-byte
// vectors, four loads in flight per thread.
__global__ void __launch_bounds__(256) copy_blocks_kernel(const CopyBlocksParams p) {
    griddep_wait();
    griddep_launch();
    const int pair = blockIdx.x, layer = blockIdx.y, which = blockIdx.z;
    const int64_t src = p.block_mapping[2 * (int64_t)pair];
    const int64_t dst = p.block_mapping[2 * (int64_t)pair + 1];
    if (src < 0 || src >= p.num_blocks || dst < 0 || dst >= p.num_blocks) {
        if (threadIdx.x == 0 && layer == 0 && which == 0) flag_error(p.errors, PKV_DEVERR_COPY_ID);
        return;
    }
    if (pair_conflicts(p.block_mapping, p.num_pairs, pair, src, dst, true)) {
        if (threadIdx.x == 0 && layer == 0 && which == 0) flag_error(p.errors, PKV_DEVERR_COPY_OVERLAP);
        return;
    }
    unsigned char* base = static_cast<unsigned char*>(which ? p.v[layer] : p.k[layer]);
    const uint4* s = reinterpret_cast<const uint4*>(base + src * p.block_bytes);
    uint4* d = reinterpret_cast<uint4*>(base + dst * p.block_bytes);
    const int64_t n = p.block_bytes / 16;
    int64_t i = threadIdx.x;
    for (; i + 3 * blockDim.x < n; i += 4 * blockDim.x) {
        const uint4 a = s[i], b = s[i + blockDim.x], c = s[i + 2 * blockDim.x],
                    e = s[i + 3 * blockDim.x];
        d[i] = a;
        d[i + blockDim.x] = b;
        d[i + 2 * blockDim.x] = c;
        d[i + 3 * blockDim.x] = e;
    }
    for (; i < n; i += blockDim.x) d[i] = s[i];
}

// Swap between a device pool and a pinned host pool (either direction): the
// host side is read or written in place through unified addressing, so a
// swap of scattered blocks is one launch.  grid = (pairs, caches); each CTA
// moves one block with 16-byte vectors, eight loads in flight per thread to
// cover the host link's latency.
__global__ void __launch_bounds__(256) swap_blocks_kernel(const SwapBlocksParams p) {
    griddep_wait();
    griddep_launch();
    const int pair = blockIdx.x, c = blockIdx.y;
    const int64_t src = p.block_mapping[2 * (int64_t)pair];
    const int64_t dst = p.block_mapping[2 * (int64_t)pair + 1];
    if (src < 0 || src >= p.src_blocks || dst < 0 || dst >= p.dst_blocks) {
        if (threadIdx.x == 0 && c == 0) flag_error(p.errors, PKV_DEVERR_COPY_ID);
        return;
    }
    if (pair_conflicts(p.block_mapping, p.num_pairs, pair, src, dst, false)) {
        if (threadIdx.x == 0 && c == 0) flag_error(p.errors, PKV_DEVERR_COPY_OVERLAP);
        return;
    }
    const uint4* s = reinterpret_cast<const uint4*>(static_cast<const unsigned char*>(p.src[c]) +
                                                    src * p.block_bytes);
    uint4* d = reinterpret_cast<uint4*>(static_cast<unsigned char*>(p.dst[c]) + dst * p.block_bytes);
    const int64_t n = p.block_bytes / 16;
    int64_t i = threadIdx.x;
    constexpr int U = 8;
    for (; i + (U - 1) * (int64_t)blockDim.x < n; i += U * (int64_t)blockDim.x) {
        uint4 v[U];
#pragma unroll
        for (int k = 0; k < U; ++k) v[k] = s[i + k * blockDim.x];
#pragma unroll
        for (int k = 0; k < U; ++k) d[i + k * blockDim.x] = v[k];
    }
    for (; i < n; i += blockDim.x) d[i] = s[i];
}

cudaError_t launch_swap_blocks(const SwapBlocksParams& p, int num_pairs, int num_caches,
                               cudaStream_t stream) {
    if (num_pairs == 0 || num_caches == 0) return cudaSuccess;
    return launch_pdl(swap_blocks_kernel, dim3(num_pairs, num_caches), dim3(256), 0, stream, p);
}

// Cache write into an FP8 (E4M3) cache: each element becomes
// e4m3(x / scale) -- the quotient correctly rounded in fp32, then rounded to
// nearest-even E4M3 with saturation at +-448.  One thread per 16 output
// bytes (16 elements) of one (token, KV head) row.
template <typename TS>
__global__ void reshape_and_cache_fp8_kernel(const CacheWriteFp8Params p) {
    griddep_wait();
    griddep_launch();
    constexpr int EPS = Elem<TS>::kPerChunk;      // source elements per 16 bytes
    const int64_t chunks_per_row = p.head_size / 16;
    const int64_t per_token = (int64_t)p.num_kv_heads * chunks_per_row;
    const int64_t total = (int64_t)p.num_tokens * per_token;
    const int64_t pool_slots = (int64_t)p.num_blocks * p.block_size;
    for (int64_t w = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; w < total;
         w += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = w / per_token;
        const int64_t rem = w - i * per_token;
        const int64_t g = rem / chunks_per_row;
        const int64_t ch = rem - g * chunks_per_row;
        const int64_t slot = p.slot_mapping[i];
        if (slot < 0) continue;
        if (slot >= pool_slots) {
            if (rem == 0) flag_error(p.errors, PKV_DEVERR_SLOT);
            continue;
        }
        const int64_t blk = slot / p.block_size, off = slot - blk * p.block_size;
        const int64_t dst = ((blk * p.num_kv_heads + g) * p.block_size + off) * p.head_size + ch * 16;
#pragma unroll
        for (int which = 0; which < 2; ++which) {
            const TS* src = reinterpret_cast<const TS*>(which ? p.value : p.key) +
                            i * (which ? p.value_stride : p.key_stride) + g * p.head_size + ch * 16;
            const float sc = which ? p.v_scale : p.k_scale;
            float x[16];
#pragma unroll
            for (int k = 0; k < 16 / EPS; ++k)
                Elem<TS>::widen(reinterpret_cast<const uint4*>(src)[k], x + k * EPS);
            uint32_t out[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint16_t lo = f32x2_to_e4m3x2(__fdiv_rn(x[4 * k], sc), __fdiv_rn(x[4 * k + 1], sc));
                const uint16_t hi = f32x2_to_e4m3x2(__fdiv_rn(x[4 * k + 2], sc), __fdiv_rn(x[4 * k + 3], sc));
                out[k] = (uint32_t)lo | ((uint32_t)hi << 16);
            }
            *reinterpret_cast<uint4*>((which ? p.v_cache : p.k_cache) + dst) =
                make_uint4(out[0], out[1], out[2], out[3]);
        }
    }
}

cudaError_t launch_reshape_and_cache_fp8(const CacheWriteFp8Params& p, int num_sms,
                                         cudaStream_t stream) {
    const int64_t total = (int64_t)p.num_tokens * p.num_kv_heads * (p.head_size / 16);
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    int64_t blocks = (total + threads - 1) / threads;
    const int64_t cap = (int64_t)num_sms * 16;
    if (blocks > cap) blocks = cap;
    const dim3 grid((unsigned)blocks), block(threads);
    switch (p.src_dtype) {
        case PKV_F32: return launch_pdl(reshape_and_cache_fp8_kernel<float>, grid, block, 0, stream, p);
        case PKV_F16: return launch_pdl(reshape_and_cache_fp8_kernel<__half>, grid, block, 0, stream, p);
        default: return launch_pdl(reshape_and_cache_fp8_kernel<__nv_bfloat16>, grid, block, 0, stream, p);
    }
}

cudaError_t launch_reshape_and_cache(const CacheWriteParams& p, int num_sms, cudaStream_t stream) {
    const int64_t total = (int64_t)p.num_tokens * p.num_kv_heads * (p.row_bytes / 16);
    if (total == 0) return cudaSuccess;
    const int threads = 256;
    int64_t blocks = (total + threads - 1) / threads;
    const int64_t cap = (int64_t)num_sms * 16;
    if (blocks > cap) blocks = cap;
    return launch_pdl(reshape_and_cache_kernel, dim3((unsigned)blocks), dim3(threads), 0, stream, p);
}

cudaError_t launch_copy_blocks(const CopyBlocksParams& p, int num_pairs, int num_layers,
                               cudaStream_t stream) {
    if (num_pairs == 0 || num_layers == 0) return cudaSuccess;
    dim3 grid(num_pairs, num_layers, 2);
    return launch_pdl(copy_blocks_kernel, grid, dim3(256), 0, stream, p);
}

}  // namespace pkv
