// C-ABI entry points: argument checks on the host, launch planning, and the
// sticky device-check flag.  Nothing here allocates device memory.
#include <atomic>
#include <cmath>
#include <cstring>

#include "cache_ops.cuh"
#include "decode_launch.cuh"
#include "decode_tc.cuh"
#include "pagedkv.h"
#include "prefill.cuh"

#ifndef PKV_FP8_WCAP
#define PKV_FP8_WCAP 16
#endif
#ifndef PKV_FP8_RMAX
#define PKV_FP8_RMAX 3
#endif

namespace {

__device__ unsigned int g_device_errors;

constexpr int kMaxSeqs = 16384;
constexpr size_t kSchedBytes = 256;

// Polls after which a kernel's bounded wait gives up (pkv_set_wait_limit).
std::atomic<uint32_t> g_wait_limit{pkv::kWaitLimit};

struct DeviceInfo {
    std::atomic<int> sms{0};
    std::atomic<unsigned int*> errors{nullptr};
};
DeviceInfo g_devices[pkv::kMaxDevices];

// SM count and device address of the error flag for the current device.
pkv_status device_info(int* sms, unsigned int** errors) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= pkv::kMaxDevices)
        return PKV_ERR_CUDA;
    DeviceInfo& d = g_devices[dev];
    int n = d.sms.load(std::memory_order_acquire);
    unsigned int* e = d.errors.load(std::memory_order_acquire);
    if (n == 0 || e == nullptr) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return PKV_ERR_CUDA;
        void* addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_device_errors) != cudaSuccess) return PKV_ERR_CUDA;
        e = static_cast<unsigned int*>(addr);
        d.sms.store(n, std::memory_order_release);
        d.errors.store(e, std::memory_order_release);
    }
    *sms = n;
    *errors = e;
    return PKV_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int elem_bytes(pkv_dtype t) { return t == PKV_F32 ? 4 : 2; }

// Query-head columns of one decode work item: the group padded to 1, 2, 4 or
// 8 (a larger group runs as ceil(G / 8) slices of 8).
int padded_group(int g) { return g <= 1 ? 1 : g <= 2 ? 2 : g <= 4 ? 4 : 8; }

// Shape checks shared by the workspace query and the launch.
pkv_status check_shape(int num_seqs, int num_heads, int num_kv_heads, int head_size,
                       int block_size, int max_context_len, int dtype) {
    if (num_seqs <= 0 || num_heads <= 0 || num_kv_heads <= 0 || max_context_len < 0)
        return PKV_ERR_INVALID_ARG;
    if (dtype != PKV_F32 && dtype != PKV_F16 && dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
    if (head_size != 64 && head_size != 128) return PKV_ERR_UNSUPPORTED;
    if (block_size != 16 && block_size != 32) return PKV_ERR_UNSUPPORTED;
    if (num_heads % num_kv_heads != 0) return PKV_ERR_UNSUPPORTED;
    if (num_seqs > kMaxSeqs) return PKV_ERR_UNSUPPORTED;
    return PKV_OK;
}

// Tokens per partition.  Requested sizes must be multiples of block_size and
// at most 32 blocks (one block-table entry per lane).  The library's choice
// (requested == 0) is a range: the kernel picks, per call, a block multiple
// between half and all of 16 blocks (32 for groups of 4 or more query heads,
// whose partial results are larger) so that the last round of work items
// keeps the warps busy.  Returns the smallest size the call may use (which
// sizes the workspace) and, through *largest, the largest.
int resolve_partition(int num_heads, int num_kv_heads, int block_size, int max_context_len,
                      int requested, int* largest = nullptr) {
    (void)max_context_len;
    const int cap = 32 * block_size;
    if (requested != 0) {
        if (requested < 0 || requested % block_size != 0 || requested > cap) return 0;
        if (largest) *largest = requested;
        return requested;
    }
    // the library's range: [lo, hi] blocks, chosen per call on the device;
    // lo sizes the workspace (the most partitions)
    const int G = num_heads / num_kv_heads;
    const int lo = (G >= 4 ? 16 : 8) * block_size, hi = (G >= 4 ? 64 : 16) * block_size;
    if (largest) *largest = hi;
    return lo;
}

struct WorkspaceLayout {
    size_t prefix, part_ml, part_acc, total;
    int max_parts;
};

// Whether a plain decode call takes the tensor-core split-context kernel:
// 16-bit q and caches, at least kDecodeTcMinGroup query heads per KV head,
// and the library's choice of partitions.
bool use_decode_tc(int num_heads, int num_kv_heads, int dtype, int partition_size) {
    return dtype != PKV_F32 && num_heads / num_kv_heads >= pkv::kDecodeTcMinGroup && partition_size == 0;
}

WorkspaceLayout workspace_layout(int num_seqs, int num_heads, int num_kv_heads, int head_size,
                                 int max_context_len, int ps, bool tc = false) {
    WorkspaceLayout w;
    const int ctx = max_context_len > 0 ? max_context_len : 1;
    w.max_parts = (ctx + ps - 1) / ps;
    size_t rows = w.max_parts > 1 ? (size_t)num_seqs * w.max_parts * num_heads : 0;   // partial rows
    if (tc) rows = pkv::decode_tc_partial_rows(num_seqs, num_heads, num_kv_heads);
    w.prefix = kSchedBytes;
    size_t off = round_up(w.prefix + sizeof(int32_t) * (num_seqs + 1), 256);
    w.part_ml = off;
    off = round_up(off + rows * sizeof(float2), 256);
    w.part_acc = off;
    off = round_up(off + rows * head_size * sizeof(float), 256);
    w.total = off;
    return w;
}

uint32_t warp_smem(pkv_dtype t, bool fp8_cache, int D, int BS, int G, int R) {
    if (fp8_cache) {
        switch (t) {
            case PKV_F32: return pkv::warp_smem_f32_fp8(D, BS, G, R);
            case PKV_F16: return pkv::warp_smem_f16_fp8(D, BS, G, R);
            default: return pkv::warp_smem_bf16_fp8(D, BS, G, R);
        }
    }
    switch (t) {
        case PKV_F32: return pkv::warp_smem_f32(D, BS, G, R);
        case PKV_F16: return pkv::warp_smem_f16(D, BS, G, R);
        default: return pkv::warp_smem_bf16(D, BS, G, R);
    }
}

}  // namespace

extern "C" {

const char* pkv_status_string(pkv_status s) {
    switch (s) {
        case PKV_OK: return "ok";
        case PKV_ERR_INVALID_ARG: return "invalid argument";
        case PKV_ERR_UNSUPPORTED: return "unsupported configuration";
        case PKV_ERR_CUDA: return "CUDA error";
        case PKV_ERR_OUT_OF_BLOCKS: return "out of blocks";
        case PKV_ERR_NOT_FOUND: return "unknown or duplicate sequence id";
        case PKV_ERR_WORKSPACE: return "workspace missing or too small";
        case PKV_ERR_DEVICE_CHECK: return "a device-side check fired";
    }
    return "unknown status";
}

const char* pkv_version(void) { return "pagedkv 0.1 sm_100a"; }

int paged_attention_partition_size(int num_heads, int num_kv_heads, int block_size,
                                   int max_context_len, int partition_size) {
    if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads) return 0;
    if (block_size != 16 && block_size != 32) return 0;
    return resolve_partition(num_heads, num_kv_heads, block_size, max_context_len, partition_size);
}

size_t paged_attention_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                      int head_size, int block_size, int max_context_len,
                                      pkv_dtype dtype, int partition_size) {
    if (check_shape(num_seqs, num_heads, num_kv_heads, head_size, block_size, max_context_len,
                    dtype) != PKV_OK)
        return 0;
    const int ps = resolve_partition(num_heads, num_kv_heads, block_size, max_context_len,
                                     partition_size);
    if (ps == 0) return 0;
    // room for either decode kernel (the fused and FP8 variants take the CUDA-core one)
    const size_t a = workspace_layout(num_seqs, num_heads, num_kv_heads, head_size, max_context_len, ps).total;
    if (!use_decode_tc(num_heads, num_kv_heads, dtype, partition_size)) return a;
    const size_t b =
        workspace_layout(num_seqs, num_heads, num_kv_heads, head_size, max_context_len, ps, true).total;
    return a > b ? a : b;
}

pkv_status paged_attention_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
    if (!workspace || workspace_bytes < kSchedBytes) return PKV_ERR_WORKSPACE;
    if (cudaMemsetAsync(workspace, 0, kSchedBytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return PKV_ERR_CUDA;
    return PKV_OK;
}

}  // extern "C"

namespace {

// The fused cache write of paged_attention_decode_append (null: none).
struct AppendArgs {
    const void* key;
    const void* value;
    const int64_t* slot_mapping;
    int64_t key_stride, value_stride;
};

pkv_status decode_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* block_tables, const int32_t* context_lens, float scale,
                       int num_kv_heads, int block_size, int num_seqs, int num_heads,
                       int head_size, int num_blocks, int max_blocks_per_seq, int max_context_len,
                       pkv_dtype dtype, int partition_size, void* workspace,
                       size_t workspace_bytes, void* stream, const AppendArgs* app,
                       bool fp8_cache = false, float k_scale = 1.f, float v_scale = 1.f) {
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens)
        return PKV_ERR_INVALID_ARG;
    pkv_status st = check_shape(num_seqs, num_heads, num_kv_heads, head_size, block_size,
                                max_context_len, dtype);
    if (st != PKV_OK) return st;
    if (num_blocks <= 0 || max_blocks_per_seq <= 0) return PKV_ERR_INVALID_ARG;
    if ((int64_t)max_context_len > (int64_t)max_blocks_per_seq * block_size) return PKV_ERR_INVALID_ARG;
    if (max_context_len == 0) max_context_len = max_blocks_per_seq * block_size;   // the table's bound
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned4(block_tables) || !aligned4(context_lens))
        return PKV_ERR_INVALID_ARG;
    if (!(scale == scale) || !(k_scale > 0.f) || !(v_scale > 0.f)) return PKV_ERR_INVALID_ARG;
    int ps_hi = 0;
    const int ps = resolve_partition(num_heads, num_kv_heads, block_size, max_context_len,
                                     partition_size, &ps_hi);
    if (ps == 0) return PKV_ERR_INVALID_ARG;
    // over an FP8 cache the warps retire blocks twice as fast, so longer
    // partitions leave too few items per warp: at most 32 blocks there
    if (fp8_cache && ps_hi > 32 * block_size) ps_hi = 32 * block_size;
    const bool tc = !fp8_cache && app == nullptr && use_decode_tc(num_heads, num_kv_heads, dtype, partition_size);
    const WorkspaceLayout wl =
        workspace_layout(num_seqs, num_heads, num_kv_heads, head_size, max_context_len, ps, tc);
    if (!workspace || !aligned16(workspace) || workspace_bytes < wl.total) return PKV_ERR_WORKSPACE;

    int sms = 0;
    unsigned int* errors = nullptr;
    if ((st = device_info(&sms, &errors)) != PKV_OK) return st;

    unsigned char* ws = static_cast<unsigned char*>(workspace);
    if (tc) {
        pkv::DecodeTcArgs a;
        std::memset(&a, 0, sizeof a);
        a.out = out;
        a.q = q;
        a.k_cache = k_cache;
        a.v_cache = v_cache;
        a.block_tables = block_tables;
        a.context_lens = context_lens;
        a.errors = errors;
        a.prefix = reinterpret_cast<int32_t*>(ws + wl.prefix);
        a.part_acc = reinterpret_cast<float*>(ws + wl.part_acc);
        a.part_ml = reinterpret_cast<float2*>(ws + wl.part_ml);
        a.scale = scale;
        a.num_seqs = num_seqs;
        a.num_heads = num_heads;
        a.num_kv_heads = num_kv_heads;
        a.head_size = head_size;
        a.block_size = block_size;
        a.num_blocks = num_blocks;
        a.max_blocks_per_seq = max_blocks_per_seq;
        a.max_context_len = max_context_len;
        a.dtype = dtype;
        a.wait_limit = g_wait_limit.load(std::memory_order_relaxed);
        return pkv::launch_decode_tc(a, static_cast<cudaStream_t>(stream));
    }

    const int Greal = num_heads / num_kv_heads;
    const int G = padded_group(Greal);              // kernel columns per item
    const int slices = (Greal + G - 1) / G;
    // Shared memory: per-CTA lengths and prefix sums, then one ring per warp.
    const uint32_t seq_smem = (uint32_t)round_up(sizeof(int32_t) * (2 * (size_t)num_seqs + 1), 128);
    // Eight consumer warps per SM hide the per-block latency of the consumer
    // math for 16-bit caches (measured: six warps lose 10%, ten or twelve
    // gain nothing); a ring of two stages per warp then keeps enough bytes
    // in flight.  Use the deepest ring (up to 4) that still fits eight
    // warps, else fewer warps with two stages.
    // An FP8 cache halves the bytes per element, so each warp must retire
    // blocks twice as fast: it gets more consumer warps (up to
    // PKV_FP8_WCAP) and the ring depth that lets that many fit.
    // (the FP8 tensor-core consumer serves 16-bit q; fp32 q over an FP8
    // cache takes the fp32 consumer with up to 12 warps)
    const bool fp8_mma = fp8_cache && dtype != PKV_F32;
    const int want = fp8_mma ? PKV_FP8_WCAP : (fp8_cache ? 12 : 8);
    int R = fp8_mma ? PKV_FP8_RMAX : 4;
    uint32_t per_warp = warp_smem(dtype, fp8_cache, head_size, block_size, G, R);
    while (R > 2 && (pkv::kMaxDynSmem - seq_smem) / per_warp < (uint32_t)want) {
        --R;
        per_warp = warp_smem(dtype, fp8_cache, head_size, block_size, G, R);
    }
    int W = (int)((pkv::kMaxDynSmem - seq_smem) / per_warp);
    if (W > want) W = want;
    if (fp8_mma && 32 * W > PKV_FP8_THREADS) W = PKV_FP8_THREADS / 32;
    if (W < 1) return PKV_ERR_UNSUPPORTED;

    pkv::DecodeParams p{};
    p.out = out;
    p.q = q;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.part_acc = reinterpret_cast<float*>(ws + wl.part_acc);
    p.part_ml = reinterpret_cast<float2*>(ws + wl.part_ml);
    p.sched = reinterpret_cast<int32_t*>(ws);
    p.prefix_out = reinterpret_cast<int32_t*>(ws + wl.prefix);
    p.errors = errors;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.num_seqs = num_seqs;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.num_blocks = num_blocks;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.max_context_len = max_context_len;
    // one partition fits every context: no choice to make
    p.partition_size = (wl.max_parts > 1) ? ps_hi : ps;
    p.partition_min = (wl.max_parts > 1 && ps_hi != ps) ? ps : 0;
    if (app) {
        p.key = app->key;
        p.value = app->value;
        p.slot_mapping = app->slot_mapping;
        p.key_stride = app->key_stride;
        p.value_stride = app->value_stride;
    }
    p.group = Greal;
    p.slices = slices;
    p.wait_limit = g_wait_limit.load(std::memory_order_relaxed);
    p.stages = R;
    p.warps = W;
    p.warp_smem = per_warp;
    p.seq_smem = seq_smem;

    const size_t max_items = (size_t)num_seqs * wl.max_parts * num_kv_heads * slices;
    size_t ctas = (max_items + W - 1) / W;
    if (ctas > (size_t)sms) ctas = sms;
    const size_t smem = seq_smem + (size_t)W * per_warp;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    const dim3 grid(ctas), block(32 * W);
    if (fp8_cache) {
        switch (dtype) {
            case PKV_F32: e = pkv::decode_f32_fp8(p, head_size, block_size, G, grid, block, smem, s); break;
            case PKV_F16: e = pkv::decode_f16_fp8(p, head_size, block_size, G, grid, block, smem, s); break;
            default: e = pkv::decode_bf16_fp8(p, head_size, block_size, G, grid, block, smem, s); break;
        }
    } else {
        switch (dtype) {
            case PKV_F32: e = pkv::decode_f32(p, head_size, block_size, G, grid, block, smem, s); break;
            case PKV_F16: e = pkv::decode_f16(p, head_size, block_size, G, grid, block, smem, s); break;
            default: e = pkv::decode_bf16(p, head_size, block_size, G, grid, block, smem, s); break;
        }
    }
    if (e != cudaSuccess) return PKV_ERR_CUDA;
    if (wl.max_parts > 1) {
        pkv::ReduceParams r{};   // zero: no fixed-stride layout (prefix sums)
        r.out = out;
        r.part_acc = p.part_acc;
        r.part_ml = p.part_ml;
        r.prefix = p.prefix_out;
        r.num_seqs = num_seqs;
        r.num_heads = num_heads;
        r.num_kv_heads = num_kv_heads;
        r.max_parts = wl.max_parts;
        switch (dtype) {
            case PKV_F32: e = pkv::merge_f32(r, head_size, s); break;
            case PKV_F16: e = pkv::merge_f16(r, head_size, s); break;
            default: e = pkv::merge_bf16(r, head_size, s); break;
        }
        if (e != cudaSuccess) return PKV_ERR_CUDA;
    }
    return PKV_OK;
}

}  // namespace

extern "C" {

pkv_status paged_attention_decode(void* out, const void* q, const void* k_cache,
                                  const void* v_cache, const int32_t* block_tables,
                                  const int32_t* context_lens, float scale, int num_kv_heads,
                                  int block_size, int num_seqs, int num_heads, int head_size,
                                  int num_blocks, int max_blocks_per_seq, int max_context_len,
                                  pkv_dtype dtype, int partition_size, void* workspace,
                                  size_t workspace_bytes, void* stream) {
    return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads,
                       block_size, num_seqs, num_heads, head_size, num_blocks, max_blocks_per_seq,
                       max_context_len, dtype, partition_size, workspace, workspace_bytes, stream,
                       nullptr);
}

pkv_status paged_attention_decode_fp8kv(void* out, const void* q, const void* k_cache,
                                        const void* v_cache, const int32_t* block_tables,
                                        const int32_t* context_lens, float scale, float k_scale,
                                        float v_scale, int num_kv_heads, int block_size,
                                        int num_seqs, int num_heads, int head_size, int num_blocks,
                                        int max_blocks_per_seq, int max_context_len,
                                        pkv_dtype dtype, int partition_size, void* workspace,
                                        size_t workspace_bytes, void* stream) {
    return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads,
                       block_size, num_seqs, num_heads, head_size, num_blocks, max_blocks_per_seq,
                       max_context_len, dtype, partition_size, workspace, workspace_bytes, stream,
                       nullptr, true, k_scale, v_scale);
}

pkv_status paged_attention_decode_append(void* out, const void* q, const void* key,
                                         const void* value, void* k_cache, void* v_cache,
                                         const int64_t* slot_mapping, const int32_t* block_tables,
                                         const int32_t* context_lens, float scale,
                                         int num_kv_heads, int block_size, int num_seqs,
                                         int num_heads, int head_size, int num_blocks,
                                         int max_blocks_per_seq, int max_context_len,
                                         int64_t key_token_stride, int64_t value_token_stride,
                                         pkv_dtype dtype, int partition_size, void* workspace,
                                         size_t workspace_bytes, void* stream) {
    if (!key || !value || !slot_mapping) return PKV_ERR_INVALID_ARG;
    if (!aligned16(key) || !aligned16(value) || (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
        return PKV_ERR_INVALID_ARG;
    const int64_t eb = elem_bytes(dtype);
    if (key_token_stride < (int64_t)num_kv_heads * head_size ||
        value_token_stride < (int64_t)num_kv_heads * head_size ||
        (key_token_stride * eb) % 16 || (value_token_stride * eb) % 16)
        return PKV_ERR_INVALID_ARG;
    const AppendArgs app{key, value, slot_mapping, key_token_stride, value_token_stride};
    return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads,
                       block_size, num_seqs, num_heads, head_size, num_blocks, max_blocks_per_seq,
                       max_context_len, dtype, partition_size, workspace, workspace_bytes, stream,
                       &app);
}

pkv_status reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                             const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                             int head_size, int block_size, int num_blocks,
                             int64_t key_token_stride, int64_t value_token_stride,
                             pkv_dtype dtype, void* stream) {
    if (num_tokens < 0 || num_kv_heads <= 0 || head_size <= 0 || block_size <= 0 || num_blocks <= 0)
        return PKV_ERR_INVALID_ARG;
    if (dtype != PKV_F32 && dtype != PKV_F16 && dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PKV_OK;
    if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PKV_ERR_INVALID_ARG;
    const int eb = elem_bytes(dtype);
    const int64_t row = (int64_t)head_size * eb;
    if (row % 16 != 0) return PKV_ERR_UNSUPPORTED;
    if (key_token_stride < (int64_t)num_kv_heads * head_size ||
        value_token_stride < (int64_t)num_kv_heads * head_size)
        return PKV_ERR_INVALID_ARG;
    if ((key_token_stride * eb) % 16 || (value_token_stride * eb) % 16) return PKV_ERR_INVALID_ARG;
    if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
        return PKV_ERR_INVALID_ARG;
    int sms = 0;
    unsigned int* errors = nullptr;
    pkv_status st = device_info(&sms, &errors);
    if (st != PKV_OK) return st;
    pkv::CacheWriteParams p{};
    p.key = static_cast<const unsigned char*>(key);
    p.value = static_cast<const unsigned char*>(value);
    p.k_cache = static_cast<unsigned char*>(k_cache);
    p.v_cache = static_cast<unsigned char*>(v_cache);
    p.slot_mapping = slot_mapping;
    p.errors = errors;
    p.key_stride_bytes = key_token_stride * eb;
    p.value_stride_bytes = value_token_stride * eb;
    p.row_bytes = row;
    p.num_tokens = num_tokens;
    p.num_kv_heads = num_kv_heads;
    p.block_size = block_size;
    p.num_blocks = num_blocks;
    if (pkv::launch_reshape_and_cache(p, sms, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return PKV_ERR_CUDA;
    return PKV_OK;
}

pkv_status reshape_and_cache_fp8kv(const void* key, const void* value, void* k_cache,
                                  void* v_cache, const int64_t* slot_mapping, int num_tokens,
                                  int num_kv_heads, int head_size, int block_size, int num_blocks,
                                  int64_t key_token_stride, int64_t value_token_stride,
                                  pkv_dtype dtype, float k_scale, float v_scale, void* stream) {
    if (num_tokens < 0 || num_kv_heads <= 0 || block_size <= 0 || num_blocks <= 0)
        return PKV_ERR_INVALID_ARG;
    if (dtype != PKV_F32 && dtype != PKV_F16 && dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
    if (head_size != 64 && head_size != 128) return PKV_ERR_UNSUPPORTED;
    if (!(k_scale > 0.f) || !(v_scale > 0.f)) return PKV_ERR_INVALID_ARG;
    if (num_tokens == 0) return PKV_OK;
    if (!key || !value || !k_cache || !v_cache || !slot_mapping) return PKV_ERR_INVALID_ARG;
    const int eb = elem_bytes(dtype);
    if (key_token_stride < (int64_t)num_kv_heads * head_size ||
        value_token_stride < (int64_t)num_kv_heads * head_size ||
        (key_token_stride * eb) % 16 || (value_token_stride * eb) % 16)
        return PKV_ERR_INVALID_ARG;
    if (!aligned16(key) || !aligned16(value) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
        return PKV_ERR_INVALID_ARG;
    int sms = 0;
    unsigned int* errors = nullptr;
    pkv_status st = device_info(&sms, &errors);
    if (st != PKV_OK) return st;
    pkv::CacheWriteFp8Params p{};
    p.key = key;
    p.value = value;
    p.k_cache = static_cast<unsigned char*>(k_cache);
    p.v_cache = static_cast<unsigned char*>(v_cache);
    p.slot_mapping = slot_mapping;
    p.errors = errors;
    p.key_stride = key_token_stride;
    p.value_stride = value_token_stride;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.num_tokens = num_tokens;
    p.num_kv_heads = num_kv_heads;
    p.head_size = head_size;
    p.block_size = block_size;
    p.num_blocks = num_blocks;
    p.src_dtype = dtype;
    if (pkv::launch_reshape_and_cache_fp8(p, sms, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return PKV_ERR_CUDA;
    return PKV_OK;
}

pkv_status copy_blocks(void* const* k_caches, void* const* v_caches, int num_layers,
                       const int64_t* block_mapping, int num_pairs, int num_blocks,
                       int64_t block_bytes, void* stream) {
    if (num_layers < 0 || num_layers > pkv::kMaxLayers || num_pairs < 0 || num_blocks <= 0 ||
        block_bytes <= 0 || block_bytes % 16 != 0)
        return PKV_ERR_INVALID_ARG;
    if (num_pairs == 0 || num_layers == 0) return PKV_OK;
    if (!k_caches || !v_caches || !block_mapping || (reinterpret_cast<uintptr_t>(block_mapping) & 7u))
        return PKV_ERR_INVALID_ARG;
    if (num_pairs > 65535 || num_layers > 65535) return PKV_ERR_UNSUPPORTED;
    pkv::CopyBlocksParams p;
    std::memset(&p, 0, sizeof p);
    for (int l = 0; l < num_layers; ++l) {
        if (!k_caches[l] || !v_caches[l] || !aligned16(k_caches[l]) || !aligned16(v_caches[l]))
            return PKV_ERR_INVALID_ARG;
        p.k[l] = k_caches[l];
        p.v[l] = v_caches[l];
    }
    int sms = 0;
    unsigned int* errors = nullptr;
    pkv_status st = device_info(&sms, &errors);
    if (st != PKV_OK) return st;
    p.block_mapping = block_mapping;
    p.errors = errors;
    p.block_bytes = block_bytes;
    p.num_blocks = num_blocks;
    p.num_pairs = num_pairs;
    if (pkv::launch_copy_blocks(p, num_pairs, num_layers, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
        return PKV_ERR_CUDA;
    return PKV_OK;
}

pkv_status swap_blocks(const void* const* src_caches, void* const* dst_caches, int num_caches,
                       const int64_t* block_mapping, int num_pairs, int src_num_blocks,
                       int dst_num_blocks, int64_t block_bytes, void* stream) {
    if (num_caches < 0 || num_caches > 2 * pkv::kMaxLayers || num_pairs < 0 || src_num_blocks <= 0 ||
        dst_num_blocks <= 0 || block_bytes <= 0 || block_bytes % 16 != 0)
        return PKV_ERR_INVALID_ARG;
    if (num_pairs == 0 || num_caches == 0) return PKV_OK;
    if (!src_caches || !dst_caches || !block_mapping || (reinterpret_cast<uintptr_t>(block_mapping) & 7u))
        return PKV_ERR_INVALID_ARG;
    if (num_pairs > 65535) return PKV_ERR_UNSUPPORTED;
    // Every buffer must be reachable from the device: device memory, or host
    // memory that is pinned (page-locked) and mapped.
    auto reachable = [](const void* ptr) {
        cudaPointerAttributes a;
        if (cudaPointerGetAttributes(&a, ptr) != cudaSuccess) {
            cudaGetLastError();
            return false;
        }
        if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) return true;
        return a.type == cudaMemoryTypeHost && a.devicePointer == ptr;
    };
    pkv::SwapBlocksParams p;
    std::memset(&p, 0, sizeof p);
    for (int c = 0; c < num_caches; ++c) {
        if (!src_caches[c] || !dst_caches[c] || !aligned16(src_caches[c]) || !aligned16(dst_caches[c]))
            return PKV_ERR_INVALID_ARG;
        if (!reachable(src_caches[c]) || !reachable(dst_caches[c])) return PKV_ERR_INVALID_ARG;
        p.src[c] = src_caches[c];
        p.dst[c] = dst_caches[c];
    }
    if (!reachable(block_mapping)) return PKV_ERR_INVALID_ARG;
    int sms = 0;
    unsigned int* errors = nullptr;
    pkv_status st = device_info(&sms, &errors);
    if (st != PKV_OK) return st;
    p.block_mapping = block_mapping;
    p.errors = errors;
    p.block_bytes = block_bytes;
    p.src_blocks = src_num_blocks;
    p.dst_blocks = dst_num_blocks;
    p.num_pairs = num_pairs;
    if (pkv::launch_swap_blocks(p, num_pairs, num_caches, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess)
        return PKV_ERR_CUDA;
    return PKV_OK;
}

pkv_status paged_attention_prefill(void* out, const void* q, const void* k_cache,
                                   const void* v_cache, const int32_t* block_tables,
                                   const int32_t* context_lens, const int32_t* query_start_loc,
                                   float scale, int num_tokens, int num_seqs, int num_heads,
                                   int num_kv_heads, int head_size, int block_size,
                                   int num_blocks, int max_blocks_per_seq, int max_query_len,
                                   pkv_dtype dtype, void* stream) {
    if (num_tokens < 0 || num_seqs <= 0 || num_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 ||
        max_blocks_per_seq <= 0 || max_query_len < 0 || max_query_len > num_tokens)
        return PKV_ERR_INVALID_ARG;
    if (dtype != PKV_F16 && dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
    if (head_size != 64 && head_size != 128) return PKV_ERR_UNSUPPORTED;
    if (block_size != 16 && block_size != 32) return PKV_ERR_UNSUPPORTED;
    if (num_heads % num_kv_heads != 0 || num_heads / num_kv_heads > pkv::kPrefillMaxGroup)
        return PKV_ERR_UNSUPPORTED;
    if ((int64_t)num_blocks * num_kv_heads * block_size >= (int64_t)0x7fffffff - block_size)
        return PKV_ERR_UNSUPPORTED;
    if (!(scale > 0.f) || !(scale < INFINITY)) return PKV_ERR_INVALID_ARG;
    if (num_tokens == 0) return PKV_OK;
    if (max_query_len == 0) return PKV_ERR_INVALID_ARG;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start_loc)
        return PKV_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
        !aligned4(block_tables) || !aligned4(context_lens) || !aligned4(query_start_loc))
        return PKV_ERR_INVALID_ARG;
    int sms = 0;
    unsigned int* errors = nullptr;
    pkv_status st = device_info(&sms, &errors);
    if (st != PKV_OK) return st;
    pkv::PrefillArgs a;
    std::memset(&a, 0, sizeof a);
    a.out = out;
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.query_start_loc = query_start_loc;
    a.errors = errors;
    a.scale = scale;
    a.num_tokens = num_tokens;
    a.num_seqs = num_seqs;
    a.num_heads = num_heads;
    a.num_kv_heads = num_kv_heads;
    a.head_size = head_size;
    a.block_size = block_size;
    a.num_blocks = num_blocks;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.max_query_len = max_query_len;
    a.dtype = dtype;
    a.wait_limit = g_wait_limit.load(std::memory_order_relaxed);
    return pkv::launch_prefill(a, static_cast<cudaStream_t>(stream));
}

pkv_status pkv_set_wait_limit(int64_t polls) {
    if (polls > (int64_t)UINT32_MAX) return PKV_ERR_INVALID_ARG;
    g_wait_limit.store(polls < 0 ? pkv::kWaitLimit : (uint32_t)polls, std::memory_order_relaxed);
    return PKV_OK;
}

pkv_status pkv_read_device_errors(void* stream, uint32_t* bits) {
    if (!bits) return PKV_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return PKV_ERR_CUDA;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_errors, sizeof v) != cudaSuccess) return PKV_ERR_CUDA;
    if (v && cudaMemcpyToSymbol(g_device_errors, &zero, sizeof zero) != cudaSuccess)
        return PKV_ERR_CUDA;
    *bits = v;
    return v ? PKV_ERR_DEVICE_CHECK : PKV_OK;
}

}  // extern "C"
