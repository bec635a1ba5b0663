// Tensor-core split-context decode: tensor maps for q and the two caches, one
// kernel instance per (element type, head size, block size), then the merge.
#include <atomic>
#include <cstring>

#include "decode_launch.cuh"
#include "decode_tc.cuh"
#include "decode_tc_kernel.cuh"
#include "tmap.cuh"

namespace pkv {
namespace {

template <typename T, int D, int BS>
pkv_status run(const DecodeTcArgs& a, cudaStream_t stream) {
    using S = DecodeTcShape<T, D, BS>;
    const CUtensorMapDataType type =
        std::is_same<T, __nv_bfloat16>::value ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const cuuint64_t esz = sizeof(T);
    const int G = a.num_heads / a.num_kv_heads;
    const int GR = G < S::M ? G : S::M;      // q rows per box
    alignas(64) CUtensorMap tm_q, tm_k, tm_v;
    {
        const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)a.num_heads, (cuuint64_t)a.num_seqs};
        const cuuint64_t strides[2] = {D * esz, (cuuint64_t)a.num_heads * D * esz};
        const cuuint32_t box[3] = {64, (cuuint32_t)GR, 1};
        if (!encode_tiled(&tm_q, type, 3, a.q, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return PKV_ERR_CUDA;
    }
    const int64_t rows = (int64_t)a.num_blocks * a.num_kv_heads * BS;
    if (rows > 0x7fffffff - BS) return PKV_ERR_UNSUPPORTED;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
        const cuuint64_t strides[1] = {D * esz};
        const cuuint32_t box[2] = {64, (cuuint32_t)BS};
        if (!encode_tiled(&tm_k, type, 2, a.k_cache, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !encode_tiled(&tm_v, type, 2, a.v_cache, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
            return PKV_ERR_CUDA;
    }
    DecodeTcParams p;
    std::memset(&p, 0, sizeof p);
    p.part_acc = a.part_acc;
    p.part_ml = a.part_ml;
    p.prefix = a.prefix;
    p.block_tables = a.block_tables;
    p.context_lens = a.context_lens;
    p.errors = a.errors;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.num_seqs = a.num_seqs;
    p.num_heads = a.num_heads;
    p.num_kv_heads = a.num_kv_heads;
    p.num_blocks = a.num_blocks;
    p.max_blocks_per_seq = a.max_blocks_per_seq;
    p.max_len = a.max_context_len < a.max_blocks_per_seq * BS ? a.max_context_len : a.max_blocks_per_seq * BS;
    p.group = G;
    p.slices = (G + S::M - 1) / S::M;
    p.rows = GR;
    p.cache_rows = (int)rows;
    p.wait_limit = a.wait_limit;
    auto kernel = paged_decode_tc_kernel<T, D, BS>;
    static std::atomic<bool> configured[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKV_ERR_CUDA;
    if (!configured[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S::SMEM) !=
            cudaSuccess)
            return PKV_ERR_CUDA;
        configured[dev].store(true, std::memory_order_release);
    }
    if (launch_pdl(kernel, dim3(kDecodeTcCtas), dim3(kDecodeTcThreads), S::SMEM, stream, p, tm_q, tm_k, tm_v) !=
        cudaSuccess)
        return PKV_ERR_CUDA;

    ReduceParams r{};
    r.out = a.out;
    r.part_acc = a.part_acc;
    r.part_ml = a.part_ml;
    r.num_seqs = a.num_seqs;
    r.num_heads = a.num_heads;
    r.num_kv_heads = a.num_kv_heads;
    r.max_parts = 2 * kDecodeTcCtas;         // a unit spans at most every CTA
    r.tc_prefix = a.prefix;
    r.tc_ctas = kDecodeTcCtas;
    r.tc_slices = p.slices;
    r.tc_rows = GR;
    r.tc_unit_cost = kTcUnitCost;
    cudaError_t e = std::is_same<T, __nv_bfloat16>::value ? merge_bf16(r, D, stream) : merge_f16(r, D, stream);
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

template <typename T, int D>
pkv_status by_block(const DecodeTcArgs& a, cudaStream_t stream) {
    switch (a.block_size) {
        case 16: return run<T, D, 16>(a, stream);
        case 32: return run<T, D, 32>(a, stream);
        default: return PKV_ERR_UNSUPPORTED;
    }
}

template <typename T>
pkv_status by_head(const DecodeTcArgs& a, cudaStream_t stream) {
    switch (a.head_size) {
        case 64: return by_block<T, 64>(a, stream);
        case 128: return by_block<T, 128>(a, stream);
        default: return PKV_ERR_UNSUPPORTED;
    }
}

}  // namespace

size_t decode_tc_partial_rows(int num_seqs, int num_heads, int num_kv_heads) {
    const int G = num_heads / num_kv_heads;
    const size_t units = (size_t)num_seqs * num_kv_heads * ((G + 127) / 128);
    return 2 * ((size_t)kDecodeTcCtas + units) * (size_t)(G < 128 ? G : 128);
}

pkv_status launch_decode_tc(const DecodeTcArgs& a, cudaStream_t stream) {
    switch (a.dtype) {
        case PKV_F16: return by_head<__half>(a, stream);
        case PKV_BF16: return by_head<__nv_bfloat16>(a, stream);
        default: return PKV_ERR_UNSUPPORTED;
    }
}

}  // namespace pkv
