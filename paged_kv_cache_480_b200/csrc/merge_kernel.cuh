// Log-sum-exp merge of split contexts: the second kernel of the partitioned
// decode.  For one sequence and query head with partitions p holding the
// unnormalised accumulator acc_p, the running max m_p (log2 units) and the
// sum l_p, the exact identity
//   M = max_p m_p,  w_p = 2^(m_p - M),  out = sum_p w_p acc_p / sum_p w_p l_p
// gives the attention over the whole context.
#pragma once

#include "common.cuh"

namespace pkv {

struct ReduceParams {
    void* out;
    const float* part_acc;     // [items][G][D]
    const float2* part_ml;     // [items][G]
    const int32_t* prefix;     // [S + 1] partitions before each sequence
    int num_seqs, num_heads, num_kv_heads;
    int max_parts;             // partitions per sequence at most
};

__device__ __forceinline__ float merge_ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// One CTA of 128 threads per (sequence, query head).  Thread = (partition
// group pg, 4 dims d4): group pg sums partitions pg, pg + NPG, ... with four
// loads in flight, then the groups add up through shared memory.  The (m, l)
// pairs are staged in shared memory first.
template <typename T, int D>
__global__ void __launch_bounds__(128) lse_merge_kernel(const ReduceParams p) {
    constexpr int TPH = D / 4;          // threads per partition group (4 dims each)
    constexpr int NPG = 128 / TPH;      // partition groups
    extern __shared__ float2 s_ml[];    // [max_parts]
    __shared__ float4 s_num[NPG][TPH];
    griddep_wait();
    const int s = blockIdx.x, h = blockIdx.y;
    const int np = p.prefix[s + 1] - p.prefix[s];
    if (np <= 1) return;                // written by the decode kernel itself
    const int G = p.num_heads / p.num_kv_heads;
    const int g = h / G, hh = h % G;
    const int base = p.prefix[s];
    for (int q = threadIdx.x; q < np; q += blockDim.x)
        s_ml[q] = p.part_ml[((size_t)(base + q) * p.num_kv_heads + g) * G + hh];
    __syncthreads();
    float M = -INFINITY, den = 0.f;
    for (int q = 0; q < np; ++q) M = fmaxf(M, s_ml[q].x);
    if (M != -INFINITY)
        for (int q = 0; q < np; ++q)
            if (s_ml[q].x != -INFINITY) den = fmaf(merge_ex2(s_ml[q].x - M), s_ml[q].y, den);

    const int pg = threadIdx.x / TPH, d4 = threadIdx.x % TPH;
    const float4* acc = reinterpret_cast<const float4*>(p.part_acc) + d4;
    const size_t stride = (size_t)p.num_kv_heads * G * TPH;           // float4s between partitions
    const size_t first = (((size_t)base * p.num_kv_heads + g) * G + hh) * TPH;
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
        for (int q0 = pg; q0 < np; q0 += 4 * NPG) {
            float4 a[4];
            float w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int q = q0 + k * NPG;
                const bool ok = q < np && s_ml[q < np ? q : 0].x != -INFINITY;
                w[k] = ok ? merge_ex2(s_ml[q].x - M) : 0.f;
                a[k] = ok ? acc[first + (size_t)q * stride] : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                num.x = fmaf(w[k], a[k].x, num.x);
                num.y = fmaf(w[k], a[k].y, num.y);
                num.z = fmaf(w[k], a[k].z, num.z);
                num.w = fmaf(w[k], a[k].w, num.w);
            }
        }
    }
    s_num[pg][d4] = num;
    __syncthreads();
    if (pg != 0) return;
    for (int k = 1; k < NPG; ++k) {
        const float4 v = s_num[k][d4];
        num.x += v.x;
        num.y += v.y;
        num.z += v.z;
        num.w += v.w;
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    const float f[4] = {num.x * inv, num.y * inv, num.z * inv, num.w * inv};
    T* o = reinterpret_cast<T*>(p.out) + ((size_t)s * p.num_heads + h) * D + d4 * 4;
#pragma unroll
    for (int e = 0; e < 4; ++e) o[e] = static_cast<T>(f[e]);
}

}  // namespace pkv
