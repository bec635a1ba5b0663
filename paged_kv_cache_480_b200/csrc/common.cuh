// Device helpers shared by the library's kernels: element traits, bulk-copy
// and mbarrier wrappers (inline PTX for sm_100a), and the sticky
// device-check flag.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "pagedkv.h"

namespace pkv {

// ---------------------------------------------------------------------------
// Element traits: 16-byte chunks of storage elements widened to fp32.
// ---------------------------------------------------------------------------
template <typename T> struct Elem;

template <> struct Elem<float> {
    static constexpr int kPerChunk = 4;
    __device__ __forceinline__ static void widen(const uint4& c, float* f) {
        f[0] = __uint_as_float(c.x);
        f[1] = __uint_as_float(c.y);
        f[2] = __uint_as_float(c.z);
        f[3] = __uint_as_float(c.w);
    }
    __device__ __forceinline__ static uint4 narrow(const float* f) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                          __float_as_uint(f[3]));
    }
};

template <> struct Elem<__nv_bfloat16> {
    static constexpr int kPerChunk = 8;
    // bf16 is the upper half of an fp32: widening is a shift / mask.
    __device__ __forceinline__ static void widen2(uint32_t w, float& lo, float& hi) {
        lo = __uint_as_float(w << 16);
        hi = __uint_as_float(w & 0xffff0000u);
    }
    __device__ __forceinline__ static void widen(const uint4& c, float* f) {
        widen2(c.x, f[0], f[1]);
        widen2(c.y, f[2], f[3]);
        widen2(c.z, f[4], f[5]);
        widen2(c.w, f[6], f[7]);
    }
    __device__ __forceinline__ static uint32_t pack2(float lo, float hi) {
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // round to nearest even
        return *reinterpret_cast<uint32_t*>(&v);
    }
    __device__ __forceinline__ static uint4 narrow(const float* f) {
        return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]),
                          pack2(f[6], f[7]));
    }
};

template <> struct Elem<__half> {
    static constexpr int kPerChunk = 8;
    __device__ __forceinline__ static void widen2(uint32_t w, float& lo, float& hi) {
        __half2 h = *reinterpret_cast<__half2*>(&w);
        float2 f = __half22float2(h);
        lo = f.x;
        hi = f.y;
    }
    __device__ __forceinline__ static void widen(const uint4& c, float* f) {
        widen2(c.x, f[0], f[1]);
        widen2(c.y, f[2], f[3]);
        widen2(c.z, f[4], f[5]);
        widen2(c.w, f[6], f[7]);
    }
    __device__ __forceinline__ static uint32_t pack2(float lo, float hi) {
        __half2 v = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&v);
    }
    __device__ __forceinline__ static uint4 narrow(const float* f) {
        return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]),
                          pack2(f[6], f[7]));
    }
};

// FP8 E4M3 cache elements (1 sign, 4 exponent bits with bias 7, 3 fraction
// bits; no infinities, 0x7f/0xff are NaN, largest finite 448).  Stored
// values are the real values divided by a per-tensor scale.
struct fp8e4m3 {
    uint8_t bits;
};

// Two E4M3 values (low byte -> low half) to two exact fp16 values.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t v) {
    uint32_t h;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(v));
    return h;
}

// Round two fp32 values to E4M3 (nearest, ties to even; beyond +-448 they
// saturate to +-448): lo -> low byte, hi -> high byte.
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float lo, float hi) {
    uint16_t v;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(v) : "f"(hi), "f"(lo));
    return v;
}

template <> struct Elem<fp8e4m3> {
    static constexpr int kPerChunk = 16;
    __device__ __forceinline__ static void widen4(uint32_t w, float* f) {
        const uint32_t ha = e4m3x2_to_f16x2((uint16_t)(w & 0xffffu));
        const uint32_t hb = e4m3x2_to_f16x2((uint16_t)(w >> 16));
        const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&ha));
        const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&hb));
        f[0] = a.x;
        f[1] = a.y;
        f[2] = b.x;
        f[3] = b.y;
    }
    __device__ __forceinline__ static void widen(const uint4& c, float* f) {
        widen4(c.x, f);
        widen4(c.y, f + 4);
        widen4(c.z, f + 8);
        widen4(c.w, f + 12);
    }
};

// ---------------------------------------------------------------------------
// Shared-memory and bulk-copy (TMA, untiled) primitives.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Orders this thread's generic-proxy shared-memory accesses before later
// async-proxy (bulk copy) accesses to the same memory.
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// One arrival that also announces `bytes` of incoming asynchronous writes.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}

// Bounded wait: gives up after `limit` polls (each poll may suspend the
// thread for a short hardware-defined time) and returns false.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint32_t limit) {
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// Global -> shared bulk copy of `bytes` (multiple of 16, both addresses
// 16-byte aligned) completing on mbarrier `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Same, with an L2 cache-policy hint (evict-first for streamed K/V).
__device__ __forceinline__ void bulk_g2s_hint(uint32_t dst, const void* src, uint32_t bytes,
                                              uint32_t bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], "
        "[%1], %2, [%3], %4;" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ int lds32(uint32_t addr) {
    int v;
    asm volatile("ld.shared.s32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ void flag_error(unsigned int* flags, unsigned int bit) {
    if (flags) atomicOr(flags, bit);
}

// Programmatic dependent launch.  Every kernel of the library is launched
// with programmatic stream serialisation: it may become resident while its
// predecessor on the stream finishes, and waits (griddep_wait) for that
// predecessor's completion and memory before touching global memory.  Each
// kernel lets its own successor get resident early (griddep_launch).
__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Polls of an mbarrier before a wait is declared lost (far beyond any
// real copy latency; keeps a broken copy from hanging the GPU).
constexpr uint32_t kWaitLimit = 1u << 22;

}  // namespace pkv
