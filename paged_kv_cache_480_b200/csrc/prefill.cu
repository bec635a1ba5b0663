// Paged prefill launch: tensor maps for q and the two caches, one kernel
// instance per (element type, head size, block size); the group size is a
// launch parameter.
#include <atomic>
#include <cstring>

#include "prefill.cuh"
#include "prefill_kernel.cuh"
#include "tmap.cuh"

namespace pkv {
namespace {

constexpr int kMaxDevices = 64;

// Item counters of the persistent prefill grid: each launch takes the next of
// kCounterSlots pairs (item counter, finished CTAs), which its last CTA
// resets to zero.  Up to kCounterSlots launches may run at the same time.
constexpr int kCounterSlots = 64;
__device__ int g_prefill_sched[2 * kCounterSlots];
std::atomic<unsigned> g_prefill_launches{0};
std::atomic<int*> g_prefill_sched_addr[kMaxDevices];

int* counter_slot(int dev) {
    int* base = g_prefill_sched_addr[dev].load(std::memory_order_acquire);
    if (base == nullptr) {
        void* addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_prefill_sched) != cudaSuccess || addr == nullptr) return nullptr;
        base = static_cast<int*>(addr);
        g_prefill_sched_addr[dev].store(base, std::memory_order_release);
    }
    return base + 2 * (g_prefill_launches.fetch_add(1, std::memory_order_relaxed) % kCounterSlots);
}

bool encode(CUtensorMap* map, CUtensorMapDataType type, int rank, const void* base, const cuuint64_t* dims,
            const cuuint64_t* strides_bytes, const cuuint32_t* box) {
    return encode_tiled(map, type, rank, base, dims, strides_bytes, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <typename T, int D, int BS>
pkv_status run(const PrefillArgs& a, cudaStream_t stream) {
    using S = PrefillShape<T, D, BS>;
    const int G = a.num_heads / a.num_kv_heads;
    if (G < 1 || G > kPrefillMaxGroup) return PKV_ERR_UNSUPPORTED;
    const int QT = S::M / G;                 // queries per query tile
    const CUtensorMapDataType type =
        std::is_same<T, __nv_bfloat16>::value ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const cuuint64_t esz = sizeof(T);
    alignas(64) CUtensorMap tm_q, tm_k, tm_v;
    {
        const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)a.num_heads, (cuuint64_t)a.num_tokens};
        const cuuint64_t strides[2] = {D * esz, (cuuint64_t)a.num_heads * D * esz};
        const cuuint32_t box[3] = {64, (cuuint32_t)G, (cuuint32_t)QT};
        if (!encode(&tm_q, type, 3, a.q, dims, strides, box)) return PKV_ERR_CUDA;
    }
    const int64_t rows = (int64_t)a.num_blocks * a.num_kv_heads * BS;
    if (rows > 0x7fffffff - BS) return PKV_ERR_UNSUPPORTED;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
        const cuuint64_t strides[1] = {D * esz};
        const cuuint32_t box[2] = {64, (cuuint32_t)BS};
        if (!encode(&tm_k, type, 2, a.k_cache, dims, strides, box)) return PKV_ERR_CUDA;
        if (!encode(&tm_v, type, 2, a.v_cache, dims, strides, box)) return PKV_ERR_CUDA;
    }
    PrefillParams p;
    std::memset(&p, 0, sizeof p);
    p.out = a.out;
    p.block_tables = a.block_tables;
    p.context_lens = a.context_lens;
    p.query_start_loc = a.query_start_loc;
    p.errors = a.errors;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.num_tokens = a.num_tokens;
    p.num_seqs = a.num_seqs;
    p.num_heads = a.num_heads;
    p.num_kv_heads = a.num_kv_heads;
    p.num_blocks = a.num_blocks;
    p.max_blocks_per_seq = a.max_blocks_per_seq;
    p.group = G;
    p.qt = QT;
    p.wait_limit = a.wait_limit;
    p.q_tiles = (a.max_query_len + 2 * QT - 1) / (2 * QT);
    p.cache_rows = (int)rows;
    int dev = 0, sms = 0, l2 = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKV_ERR_CUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev) != cudaSuccess)
        return PKV_ERR_CUDA;
    // Scheduling groups of (sequence, KV head) pairs.  Each CTA holds about
    // 1.5 items (the one it runs and the one it claimed ahead), so the K/V in
    // flight is that of (1.5 * CTAs + the group's items) / (items per pair)
    // pairs; the group is as large as keeps that within 3/4 of L2 at the
    // longest possible context, and at least 2 pairs.  Large groups let the
    // heaviest-first order inside a group balance the CTAs (whole prompts of
    // mixed lengths); small ones keep a pair's items close in time, so its
    // K/V comes from DRAM about once (chunks of long contexts).
    {
        const double pair_bytes = (double)a.max_blocks_per_seq * BS * D * sizeof(T) * 2.0;
        const double in_flight = 0.75 * l2 / (pair_bytes > 1.0 ? pair_bytes : 1.0);
        const double g = in_flight - 1.5 * sms / (p.q_tiles > 0 ? p.q_tiles : 1);
        p.sched_group = g < 2.0 ? 2 : (g > 4096.0 ? 4096 : (int)g);
    }
    const int64_t items = (int64_t)p.q_tiles * a.num_seqs * a.num_kv_heads;
    if (items > 0x7fffffff) return PKV_ERR_UNSUPPORTED;
    auto kernel = paged_prefill_kernel<T, D, BS>;
    static std::atomic<bool> configured[kMaxDevices];
    // persistent: one CTA per SM (fewer if there are fewer items)
    const int64_t grid = items < sms ? items : sms;
    p.sched = counter_slot(dev);
    if (p.sched == nullptr) return PKV_ERR_CUDA;
    if (!configured[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)S::SMEM) !=
            cudaSuccess)
            return PKV_ERR_CUDA;
        configured[dev].store(true, std::memory_order_release);
    }
    if (launch_pdl(kernel, dim3((unsigned)grid), dim3(kPrefillThreads), S::SMEM, stream, p, tm_q, tm_k,
                   tm_v) != cudaSuccess)
        return PKV_ERR_CUDA;
    return PKV_OK;
}

template <typename T, int D>
pkv_status by_block(const PrefillArgs& a, cudaStream_t stream) {
    switch (a.block_size) {
        case 16: return run<T, D, 16>(a, stream);
        case 32: return run<T, D, 32>(a, stream);
        default: return PKV_ERR_UNSUPPORTED;
    }
}

template <typename T>
pkv_status by_head(const PrefillArgs& a, cudaStream_t stream) {
    switch (a.head_size) {
        case 64: return by_block<T, 64>(a, stream);
        case 128: return by_block<T, 128>(a, stream);
        default: return PKV_ERR_UNSUPPORTED;
    }
}

}  // namespace

pkv_status launch_prefill(const PrefillArgs& a, cudaStream_t stream) {
    switch (a.dtype) {
        case PKV_F16: return by_head<__half>(a, stream);
        case PKV_BF16: return by_head<__nv_bfloat16>(a, stream);
        default: return PKV_ERR_UNSUPPORTED;
    }
}

}  // namespace pkv
