// Log-sum-exp merge of split contexts: the second kernel of the partitioned
// decode.  For one sequence and query head with partitions p holding the
// unnormalised accumulator acc_p, the running max m_p (log2 units) and the
// sum l_p, the exact identity
//   M = max_p m_p,  w_p = 2^(m_p - M),  out = sum_p w_p acc_p / sum_p w_p l_p
// gives the attention over the whole context.  Partials with m_p = -inf
// (no key) are skipped.
//
// Two layouts of the partials.  The CUDA-core decode numbers them through
// per-sequence prefix sums it publishes (a sequence with one partition wrote
// its output itself).  The tensor-core decode splits the key tiles of all
// units (sequence, KV head, slice of up to 128 query heads) into contiguous
// ranges of equal cost, one per CTA (a unit costs a fixed start cost plus its
// tiles); CTA c writes two partials (one per half) for unit u in slots
// 2 * (c + u) and 2 * (c + u) + 1, rows [slot * rows, + rows).  The CTAs
// whose range meets unit u's tiles follow from the per-sequence prefix sums
// of unit costs it publishes.
#pragma once

#include "common.cuh"

namespace pkv {

struct ReduceParams {
    void* out;
    const float* part_acc;     // [partials][H][D]
    const float2* part_ml;     // [partials][H]
    const int32_t* prefix;     // [S + 1] partitions before each sequence (CUDA-core decode)
    int num_seqs, num_heads, num_kv_heads;
    int max_parts;             // partials per sequence at most
    // tensor-core decode (tc_prefix non-null): tc_prefix[s] = the cost of one
    // unit of each sequence before s, summed (tc_unit_cost + its key tiles, 0
    // for a sequence without keys), [S] = the sum over all; tc_ctas CTAs,
    // tc_slices units per KV head, tc_rows rows per slot
    const int32_t* tc_prefix;
    int tc_ctas, tc_slices, tc_rows, tc_unit_cost;
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
    int np;
    size_t base, rs, ro;                // partial q sits at row (base + q) * rs + ro
    int64_t tc_first = 0, tc_v = 0;     // tensor-core decode: first CTA of the unit, cost of all units
    if (p.tc_prefix != nullptr) {
        const int G = p.num_heads / p.num_kv_heads;
        const int g = h / G, hh = h - g * G, sl = hh / 128;
        const int NU = p.num_kv_heads * p.tc_slices;
        const int u = g * p.tc_slices + sl;
        const int64_t w = p.tc_prefix[s + 1] - p.tc_prefix[s];     // one unit's cost
        const int64_t Ts = w > 0 ? w - p.tc_unit_cost : 0;
        tc_v = (int64_t)p.tc_prefix[p.num_seqs] * NU;
        int64_t cl = -1;
        if (Ts > 0) {
            // the CTA whose range [floor(c V / C), floor((c + 1) V / C)) holds cost index v;
            // the unit's tiles sit at [a, a + Ts)
            const int64_t C = p.tc_ctas;
            const int64_t a = (int64_t)p.tc_prefix[s] * NU + (int64_t)u * w + p.tc_unit_cost;
            tc_first = ((a + 1) * C - 1) / tc_v;
            cl = ((a + Ts) * C - 1) / tc_v;
        }
        np = 2 * (int)(cl - tc_first + 1);
        base = 2 * ((size_t)tc_first + (size_t)s * NU + u);
        rs = p.tc_rows;
        ro = hh - sl * 128;
    } else {
        np = p.prefix[s + 1] - p.prefix[s];
        if (np <= 1) return;            // written by the decode kernel itself
        base = p.prefix[s];
        rs = p.num_heads;
        ro = h;
    }
    const int pg = threadIdx.x / TPH, d4 = threadIdx.x % TPH;
    const float4* acc = reinterpret_cast<const float4*>(p.part_acc) + d4;
    const size_t stride = rs * TPH;                                   // float4s between partials
    const size_t first = (base * rs + ro) * TPH;
    // the first batch of accumulators is requested before the (m, l) pairs
    // arrive (selected once they have: a slot nobody wrote is never used)
    float4 a0[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int q = pg + k * NPG;
        a0[k] = q < np ? acc[first + (size_t)q * stride] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int q = threadIdx.x; q < np; q += blockDim.x) {
        // with fewer tiles than CTAs some CTAs' ranges are empty: they wrote nothing
        const int64_t c = tc_first + q / 2, C = p.tc_ctas;
        const bool written = p.tc_prefix == nullptr || (c + 1) * tc_v / C > c * tc_v / C;
        s_ml[q] = written ? p.part_ml[(base + q) * rs + ro] : make_float2(-INFINITY, 0.f);
    }
    __syncthreads();
    float M = -INFINITY, den = 0.f;
    for (int q = 0; q < np; ++q) M = fmaxf(M, s_ml[q].x);
    if (M != -INFINITY)
        for (int q = 0; q < np; ++q)
            if (s_ml[q].x != -INFINITY) den = fmaf(merge_ex2(s_ml[q].x - M), s_ml[q].y, den);

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
                const float4 v = q0 == pg ? a0[k] : (ok ? acc[first + (size_t)q * stride] : make_float4(0.f, 0.f, 0.f, 0.f));
                a[k] = ok ? v : make_float4(0.f, 0.f, 0.f, 0.f);
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
