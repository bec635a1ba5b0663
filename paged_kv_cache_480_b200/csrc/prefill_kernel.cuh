// Paged prefill / chunked-prefill attention on the sm_100a tensor cores
// (tcgen05 MMA, accumulators in tensor memory, operands staged by TMA).
//
// Sequence s holds L = context_lens[s] tokens in its blocks; the last n of
// them are this call's queries (rows query_start_loc[s] .. +n of q), query i
// at position L - n + i attending causally to keys 0 .. L - n + i ("PyTorch-
// CUDA-v2.9 image enables PagedAttention", workflow list: prefill writes the
// prompt's KV into pages; usage: chunked prefill).
//
// CTA = (sequence, KV head g, two query tiles of M = 128 rows each); a row
// is a (query, head-of-group) pair, row = query * G + head, so every K/V
// tile serves the G query heads that share it, and both query tiles of the
// CTA share each K/V tile brought into shared memory.  Roles:
//   warps 0-3 and 4-7  softmax of query tile 0 and 1, one row per thread
//                      (warp w reaches tensor-memory lanes 32(w%4) .. +31);
//   warp 8             issues the MMAs (one thread);
//   warp 9             streams K/V tiles through a ring of stages with TMA,
//                      refilling a stage once both tiles' PV products that
//                      read it are done.
// Per key tile j of N = 64 keys and query tile x:
//   S_x,b = Q_x K_j^T   tcgen05.mma, A = Q and B = K from 128-byte-swizzled
//                       shared memory (K-major), fp32 in tensor memory; two
//                       S buffers per query tile (b = j mod 2);
//   P     = exp2(S * scale*log2e - m_ref) rounded to the element type,
//           written over S_x,b in tensor memory;
//   O_x  += P V_j       tcgen05.mma with A = P from tensor memory and B = V
//                       from shared memory (MN-major).
// While one softmax warpgroup works, the tensor core runs the other tile's
// products.  m_ref is raised (and O and l rescaled) only when a row's maximum
// grows by more than 8 in log2 units, so O stays exact up to the final
// division by l.  Masks are applied only on tiles that reach past some row's
// position.  Every wait is bounded; the tensor memory is freed on every path.
#pragma once

#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "tc05.cuh"

namespace pkv {
namespace prefill {

constexpr unsigned kAll = 0xffffffffu;

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// ---- packed fp32 pairs (sm_100 f32x2 arithmetic) ----
__device__ __forceinline__ uint64_t f2pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2sub(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Bounded wait taken by all 32 lanes; true only if every lane saw the phase,
// so a failure leaves the whole warp on the same path.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity) {
    const bool got = mbar_wait_bounded(bar, parity, kWaitLimit);
    return __all_sync(kAll, got);
}

}  // namespace prefill

struct PrefillParams {
    void* out;                        // [T][H][D]
    const int32_t* block_tables;      // [S][MB]
    const int32_t* context_lens;      // [S]
    const int32_t* query_start_loc;   // [S + 1]
    unsigned int* errors;
    float scale_log2;                 // softmax scale * log2(e), > 0
    int num_tokens, num_seqs, num_heads, num_kv_heads, num_blocks, max_blocks_per_seq;
    int q_tiles;                      // CTAs (query-tile pairs) per (sequence, KV head)
    int cache_rows;                   // rows of the [NB * Hkv * bs][D] view of a cache
};

#ifndef PKV_PREFILL_STAGES
#define PKV_PREFILL_STAGES 4
#endif
#ifndef PKV_PREFILL_ORDER
#define PKV_PREFILL_ORDER 0
#endif


template <typename T, int D, int BS, int G>
struct PrefillShape {
    static constexpr int M = 128;               // rows per query tile
    static constexpr int QT = M / G;            // queries per query tile
    static constexpr int CQ = 2 * QT;           // queries per CTA
    static constexpr int N = 64;                // keys per tile
    static constexpr int DH = D / 64;           // 64-dim halves (one 128-byte swizzle row each)
    static constexpr int BPT = N / BS;          // cache blocks per key tile
    // K/V tiles in flight; with head size 64 the extra stages also keep a
    // second CTA (and its 512 tensor-memory columns) off the SM
    static constexpr int STAGES = D == 64 ? 6 : PKV_PREFILL_STAGES;
    static constexpr uint32_t Q_HALF = M * 128;
    static constexpr uint32_t KV_HALF = N * 128;
    static constexpr uint32_t Q_BYTES = DH * Q_HALF;        // one query tile
    static constexpr uint32_t KV_BYTES = DH * KV_HALF;      // K or V of one key tile
    static constexpr uint32_t OFF_KV = 2 * Q_BYTES;         // stage st: K at +2*st*KV_BYTES, V after
    static constexpr uint32_t OFF_BAR = OFF_KV + STAGES * 2 * KV_BYTES;
    static constexpr uint32_t SMEM = OFF_BAR + 512 + 1024;  // barriers, TMEM holder, 1 KB alignment slack
    static constexpr uint32_t TM_TILE = 256;                // columns per query tile
    static constexpr uint32_t TM_S = 0;                     // S buffers at columns 0 and N (fp32)
    static constexpr uint32_t TM_O = 2 * N;                 // O at columns 2N .. 2N + D
    static constexpr uint32_t TM_COLS = 512;
    static_assert(2 * N + D <= (int)TM_TILE, "tensor-memory budget");
    static_assert(N % BS == 0, "key tile holds whole blocks");
    static_assert(8 * (15 + 2 * STAGES) <= 256, "barrier area");
    static_assert(SMEM > 232448 / 2 && SMEM <= 232448, "one CTA per SM");
};

constexpr uint32_t kPrefillThreads = 320;

template <typename T, int D, int BS, int G>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    paged_prefill_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
    using S = PrefillShape<T, D, BS, G>;
    using namespace prefill;
    constexpr int ST = S::STAGES;
    constexpr int N = S::N;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw_s = smem_addr(smem_raw);
    const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
    unsigned char* smem = smem_raw + pad;
    const uint32_t sm = raw_s + pad;                // 1024-byte aligned shared address
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    griddep_wait();
    // ---- which queries: the later ones (more keys) are scheduled first ----
    const int Hkv = p.num_kv_heads;
    const int pairs = p.num_seqs * Hkv;
#if PKV_PREFILL_ORDER == 0
    const int tile = p.q_tiles - 1 - (int)(blockIdx.x / pairs);
    const int rest = blockIdx.x % pairs;
#else
    // the query tiles of one (sequence, KV head) run side by side and share
    // its K/V through L2
    const int tile = p.q_tiles - 1 - (int)(blockIdx.x % p.q_tiles);
    const int rest = blockIdx.x / p.q_tiles;
#endif
    const int g = rest % Hkv;
    const int s = rest / Hkv;
    const int q0 = p.query_start_loc[s];
    const int n = p.query_start_loc[s + 1] - q0;
    const int L = p.context_lens[s];
    const int i0 = tile * S::CQ;
    if (n < 0 || n > L || n > p.q_tiles * S::CQ || L > p.max_blocks_per_seq * BS || q0 < 0 ||
        q0 + n > p.num_tokens) {
        if (threadIdx.x == 0) flag_error(p.errors, PKV_DEVERR_CONTEXT);
        return;
    }
    if (i0 >= n) return;                            // whole CTA, before any barrier or TMEM use
    // key tiles each query tile needs (0: the tile holds no query)
    const int nT0 = (L - n + min(i0 + S::QT, n) + N - 1) / N;
    const int nT1 = i0 + S::QT < n ? (L - n + min(i0 + S::CQ, n) + N - 1) / N : 0;
    auto nTx = [&](int x) { return x ? nT1 : nT0; };
    const int ntiles = nT1 > 0 ? 2 : 1;
    const int nT = max(nT0, nT1);
    // the last key tile's V rows from the context end to the end of its last
    // block hold whatever the pool holds there; they are zeroed before use
    const int nblk_seq = (L + BS - 1) / BS;
    const int vz_r0 = L - (nT - 1) * N;
    const int vz_r1 = min(nblk_seq * BS - (nT - 1) * N, N);
    const bool need_vz = vz_r0 < vz_r1;

    // ---- barriers and tensor memory ----
    const uint32_t bar = sm + S::OFF_BAR;
    const uint32_t bar_q = bar;
    auto bar_full = [&](int st) { return bar + 8 * (1 + st); };                    // K/V tile landed
    auto bar_empty = [&](int st) { return bar + 8 * (1 + ST + st); };              // its PVs are done
    auto bar_s = [&](int x, int b) { return bar + 8 * (1 + 2 * ST + 6 * x + b); };   // S written
    auto bar_p = [&](int x, int b) { return bar + 8 * (3 + 2 * ST + 6 * x + b); };   // P written (128)
    auto bar_o = [&](int x, int b) { return bar + 8 * (5 + 2 * ST + 6 * x + b); };   // PV done
    const uint32_t bar_vz = bar + 8 * (13 + 2 * ST);
    const uint32_t bar_fin = bar + 8 * (14 + 2 * ST);
    uint32_t* tm_holder = reinterpret_cast<uint32_t*>(smem + S::OFF_BAR + 256);
    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int st = 0; st < ST; ++st) {
            mbar_init(bar_full(st), 1);
            mbar_init(bar_empty(st), 1);
        }
        for (int x = 0; x < 2; ++x)
            for (int b = 0; b < 2; ++b) {
                mbar_init(bar_s(x, b), 1);
                mbar_init(bar_p(x, b), 128);
                mbar_init(bar_o(x, b), 1);
            }
        mbar_init(bar_vz, 1);
        mbar_init(bar_fin, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tc05::tmem_alloc(smem_addr(tm_holder), S::TM_COLS);
        tc05::tmem_relinquish();
    }
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    const uint32_t tm = *tm_holder;

    auto q_base = [&](int x) { return sm + (uint32_t)x * S::Q_BYTES; };
    auto k_base = [&](int st) { return sm + S::OFF_KV + (uint32_t)st * 2 * S::KV_BYTES; };
    auto v_base = [&](int st) { return k_base(st) + S::KV_BYTES; };

    if (warp == 9) {
        // ===================== TMA producer =====================
        int issued = 0;
        if (lane == 0) {
            mbar_arrive_expect_tx(bar_q, ntiles * S::Q_BYTES);
            for (int x = 0; x < ntiles; ++x)
                for (int dh = 0; dh < S::DH; ++dh)
                    tc05::tma_load_3d(q_base(x) + dh * S::Q_HALF, &tm_q, dh * 64, g * G, q0 + i0 + x * S::QT,
                                      bar_q);
            for (int t = 0; t < nT; ++t) {
                const int st = t % ST;
                if (t >= ST && !mbar_wait_bounded(bar_empty(st), ((t / ST) - 1) & 1, kWaitLimit)) {
                    flag_error(p.errors, PKV_DEVERR_WAIT);
                    break;
                }
                mbar_arrive_expect_tx(bar_full(st), 2 * S::KV_BYTES);
                for (int bi = 0; bi < S::BPT; ++bi) {
                    const int lb = t * S::BPT + bi;
                    int row = p.cache_rows;                   // past the end: TMA fills zeros
                    if (lb < nblk_seq) {
                        const int phys = p.block_tables[(size_t)s * p.max_blocks_per_seq + lb];
                        if (phys >= 0 && phys < p.num_blocks) row = (phys * Hkv + g) * BS;
                        else flag_error(p.errors, PKV_DEVERR_BLOCK_ID);
                    }
                    for (int dh = 0; dh < S::DH; ++dh) {
                        const uint32_t off = dh * S::KV_HALF + bi * BS * 128;
                        tc05::tma_load_2d(k_base(st) + off, &tm_k, dh * 64, row, bar_full(st));
                        tc05::tma_load_2d(v_base(st) + off, &tm_v, dh * 64, row, bar_full(st));
                    }
                }
                issued = t + 1;
            }
            // every copy requested above lands before this warp leaves (the last
            // copy into each stage; earlier ones were consumed before their stage
            // was refilled)
            mbar_wait_bounded(bar_q, 0, kWaitLimit);
            for (int t = max(0, issued - ST); t < issued; ++t)
                mbar_wait_bounded(bar_full(t % ST), (t / ST) & 1, kWaitLimit);
        }
        issued = __shfl_sync(kAll, issued, 0);
        if (need_vz && issued == nT) {
            const int st = (nT - 1) % ST;
            if (warp_wait(bar_full(st), ((nT - 1) / ST) & 1)) {
                const int rows = vz_r1 - vz_r0;
                for (int c = lane; c < rows * S::DH * 8; c += 32) {   // 16-byte chunks
                    const int dh = c / (rows * 8);
                    const int rem = c - dh * rows * 8;
                    *reinterpret_cast<uint4*>(smem + (v_base(st) - sm) + dh * S::KV_HALF +
                                              (vz_r0 + rem / 8) * 128 + (rem % 8) * 16) = make_uint4(0u, 0u, 0u, 0u);
                }
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_vz);
            }
        }
    } else if (warp == 8) {
        // ===================== MMA issue =====================
        if (lane == 0) {
            constexpr uint32_t idesc_qk = tc05::instr_desc(kBf16, 128, N, false, false);
            constexpr uint32_t idesc_pv = tc05::instr_desc(kBf16, 128, D, false, true);
            // operand descriptors of query tile 0 and stage 0; the start-address
            // field (bits 0-13, address / 16) is advanced by plain addition
            const uint64_t dq = tc05::smem_desc(q_base(0), 16, 1024);
            const uint64_t dk = tc05::smem_desc(k_base(0), 16, 1024);
            const uint64_t dv = tc05::smem_desc(v_base(0), S::KV_HALF, 1024);
            bool ok = mbar_wait_bounded(bar_q, 0, kWaitLimit);
            for (int j = 0; ok && j <= nT; ++j) {
                if (j < nT) {                                 // S_x = Q_x K_j^T
                    const int b = j & 1, st = j % ST;
                    ok = mbar_wait_bounded(bar_full(st), (j / ST) & 1, kWaitLimit);
                    for (int x = 0; ok && x < 2; ++x) {
                        if (j >= nTx(x)) continue;
                        if (j >= 2 && !mbar_wait_bounded(bar_o(x, b), ((j - 2) >> 1) & 1, kWaitLimit)) {
                            ok = false;
                            break;
                        }
                        tc05::fence_after_sync();
                        const uint32_t d = tm + x * S::TM_TILE + S::TM_S + b * N;
                        const uint64_t ad = dq + (uint64_t)((x * S::Q_BYTES) >> 4);
                        const uint64_t bd = dk + (uint64_t)((st * 2 * S::KV_BYTES) >> 4);
                        // k-th 16-wide slice: +32 bytes inside a swizzle row, next half after 4
#pragma unroll
                        for (int k = 0; k < D / 16; ++k) {
                            const uint32_t qoff = ((k >> 2) * S::Q_HALF + (k & 3) * 32) >> 4;
                            const uint32_t koff = ((k >> 2) * S::KV_HALF + (k & 3) * 32) >> 4;
                            tc05::mma_ss(d, ad + qoff, bd + koff, idesc_qk, k > 0 ? 1u : 0u);
                        }
                        tc05::commit(bar_s(x, b));
                    }
                }
                if (ok && j >= 1) {                           // O_x += P_x V_{j-1}
                    const int jj = j - 1, b = jj & 1, st = jj % ST;
                    if (jj == nT - 1 && need_vz) ok = mbar_wait_bounded(bar_vz, 0, kWaitLimit);
                    for (int x = 0; ok && x < 2; ++x) {
                        if (jj >= nTx(x)) continue;
                        if (!mbar_wait_bounded(bar_p(x, b), (jj >> 1) & 1, kWaitLimit)) {
                            ok = false;
                            break;
                        }
                        tc05::fence_after_sync();
                        const uint32_t base = tm + x * S::TM_TILE;
                        const uint64_t vd = dv + (uint64_t)((st * 2 * S::KV_BYTES) >> 4);
                        // k-th 16 keys: 16 rows of 128 bytes further
#pragma unroll
                        for (int k = 0; k < N / 16; ++k)
                            tc05::mma_ts(base + S::TM_O, base + S::TM_S + b * N + 8 * k, vd + (uint64_t)(k * 128),
                                         idesc_pv, (jj > 0 || k > 0) ? 1u : 0u);
                        tc05::commit(bar_o(x, b));
                    }
                    if (ok) tc05::commit(bar_empty(st));
                }
            }
            if (!ok) flag_error(p.errors, PKV_DEVERR_WAIT);
            // every MMA issued above is complete before the tensor memory is freed
            tc05::commit(bar_fin);
            mbar_wait_bounded(bar_fin, 0, kWaitLimit);
        }
    } else {
        // ===================== softmax warps: one row per thread =====================
        const int x = warp >> 2;                        // query tile
        const int nTme = nTx(x);
        if (nTme > 0) {
            bool ok = true;
            const int wq = warp & 3;
            const int r = wq * 32 + lane;               // row within the tile
            const int qi = i0 + x * S::QT + r / G;      // query of this row
            const bool valid = qi < n;
            const int pos = valid ? L - n + qi : -1;    // keys 0 .. pos are visible
            const uint32_t trow = tm + x * S::TM_TILE + ((uint32_t)(wq * 32) << 16);
            const float sl2 = p.scale_log2;
            float m_ref = -INFINITY, l = 0.f;           // reference max (log2 units), sum of weights
            for (int j = 0; j < nTme; ++j) {
                const int b = j & 1;
                if (!warp_wait(bar_s(x, b), (j >> 1) & 1)) { ok = false; break; }
                tc05::fence_after_sync();
                uint32_t sv[64];
                tc05::tmem_ld32(trow + S::TM_S + b * N, *reinterpret_cast<uint32_t(*)[32]>(sv));
                tc05::tmem_ld32(trow + S::TM_S + b * N + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
                tc05::tmem_wait_ld();
                const int key0 = j * N;
                if (__any_sync(kAll, key0 + N - 1 > pos)) {      // a diagonal (or past-the-end) tile
#pragma unroll
                    for (int c = 0; c < 64; ++c)
                        if (key0 + c > pos) sv[c] = __float_as_uint(-INFINITY);
                }
                float m4[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) m4[a] = __uint_as_float(sv[a]);
#pragma unroll
                for (int c = 4; c < 64; c += 8)
#pragma unroll
                    for (int a = 0; a < 4; ++a)
                        m4[a] = max3(m4[a], __uint_as_float(sv[c + a]), __uint_as_float(sv[c + 4 + a]));
                const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
                const float mt = mx * sl2;                  // the scale is positive
                const bool raise = mt > m_ref + 8.f;
                const float new_ref = raise ? mt : m_ref;
                const float alpha = (raise && m_ref != -INFINITY) ? ex2(m_ref - new_ref) : 1.f;
                const float neg_ref = new_ref == -INFINITY ? 0.f : -new_ref;   // rows that see nothing yet
                l *= alpha;
                uint32_t pk[32];
                const uint64_t sl2x2 = f2pack(sl2, sl2), refx2 = f2pack(neg_ref, neg_ref);
                uint64_t lsum[4] = {0, 0, 0, 0};         // four packed partial sums (+0.0 bits)
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const uint64_t z = f2fma(f2pack(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1])),
                                             sl2x2, refx2);
                    float z0, z1;
                    f2unpack(z, z0, z1);
                    const float p0 = ex2(z0), p1 = ex2(z1);
                    lsum[c & 3] = f2add(lsum[c & 3], f2pack(p0, p1));
                    pk[c] = Elem<T>::pack2(p0, p1);
                }
                {
                    float a0, a1, b0, b1, c0, c1, d0, d1;
                    f2unpack(lsum[0], a0, a1);
                    f2unpack(lsum[1], b0, b1);
                    f2unpack(lsum[2], c0, c1);
                    f2unpack(lsum[3], d0, d1);
                    l += ((a0 + a1) + (b0 + b1)) + ((c0 + c1) + (d0 + d1));
                }
                // O holds PV of tiles < j: rescale rows whose reference moved (after PV(j-1) is done)
                if (j >= 1 && __any_sync(kAll, alpha != 1.f)) {
                    if (!warp_wait(bar_o(x, (j - 1) & 1), ((j - 1) >> 1) & 1)) { ok = false; break; }
                    tc05::fence_after_sync();
#pragma unroll
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t ov[32];
                        tc05::tmem_ld32(trow + S::TM_O + cc * 32, ov);
                        tc05::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                        tc05::tmem_st32(trow + S::TM_O + cc * 32, ov);
                    }
                    tc05::tmem_wait_st();
                }
                tc05::tmem_st32(trow + S::TM_S + b * N, pk);      // P over S (this row only)
                tc05::tmem_wait_st();
                tc05::fence_before_sync();
                mbar_arrive(bar_p(x, b));
                m_ref = new_ref;
            }
            // ---- epilogue: O / l to the output ----
            if (ok && warp_wait(bar_o(x, (nTme - 1) & 1), ((nTme - 1) >> 1) & 1)) {
                tc05::fence_after_sync();
                const float inv = l > 0.f ? 1.f / l : 0.f;
                T* orow = reinterpret_cast<T*>(p.out) +
                          ((size_t)(q0 + qi) * p.num_heads + (size_t)g * G + (r % G)) * D;
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t ov[32];
                    tc05::tmem_ld32(trow + S::TM_O + cc * 32, ov);
                    tc05::tmem_wait_ld();
                    if (valid) {
                        uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                w[e] = Elem<T>::pack2(__uint_as_float(ov[8 * v + 2 * e]) * inv,
                                                      __uint_as_float(ov[8 * v + 2 * e + 1]) * inv);
                            dst[v] = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    }
                }
            } else {
                ok = false;
            }
            if (!ok && lane == 0) flag_error(p.errors, PKV_DEVERR_WAIT);
        }
    }
    griddep_launch();
    tc05::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc05::fence_after_sync();
        tc05::tmem_dealloc(tm, S::TM_COLS);
    }
}

}  // namespace pkv
