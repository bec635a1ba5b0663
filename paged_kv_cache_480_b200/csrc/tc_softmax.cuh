// The softmax of one 128-key tile for the tcgen05 attention kernels (paged
// prefill and the wide-group decode): one row per thread, S in tensor memory
// as fp32 logits, P written back over S's first 64 columns as 16-bit pairs,
// O rescaled in place when a row's reference maximum moves.
//
// A row keeps a reference maximum m_ref (log2 units) and the sum l of its
// weights; P = 2^(S * scale*log2e - m_ref) rounded to the element type.  Most
// tiles keep every row's reference and take one sweep; m_ref is raised (O
// and l rescaled) only when a logit rises more than 8 above it, so O stays
// exact up to the final division by l.  A row's first tile takes the
// largest of its first 8 logits as the starting reference.  The P of keys
// 0-63 lands on S columns 0-31 and is held in registers until one warp vote
// finds no jump there (a jump redoes the tile from the intact S); keys
// 64-127 are stored at once and voted after (a jump there rescales the
// stored P and O and recomputes them from their intact S).
#pragma once

#include <math.h>

#include "common.cuh"
#include "tc05.cuh"

namespace pkv {
namespace tcsm {

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
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, uint32_t limit) {
    const bool got = mbar_wait_bounded(bar, parity, limit);
    return __all_sync(kAll, got);
}

// One tile of one row per thread.  ts / to: this warp's tensor-memory address
// of S and of O (lane field = the warp's 32 rows); key0: the tile's first key;
// keys past pos read as -inf (masked); o_valid: O holds earlier tiles' PV
// (complete: the commit the caller waited on covers them).  Leaves P in
// tensor memory (16-bit pairs over S's first 64 columns) and m_ref / l
// updated; the caller waits for the stores (tmem_wait_st) and signals P.
template <typename T, int D>
__device__ __forceinline__ void softmax_tile(uint32_t ts, uint32_t to, int key0, int pos, float sl2, bool o_valid,
                                             float& m_ref, float& l) {
    constexpr int N = 128;
    const bool diag = __any_sync(kAll, key0 + N - 1 > pos);   // a diagonal (or past-the-end) tile
    // masked keys read as -inf (their logits may be NaN past the context end)
    auto mask = [&](uint32_t (&v)[32], int col0) {
        if (diag) {
#pragma unroll
            for (int c = 0; c < 32; ++c)
                if (key0 + col0 + c > pos) v[c] = __float_as_uint(-INFINITY);
        }
    };
    // The weights of one 32-key chunk of S (16 columns of P):
    // P = 2^(S * scale*log2e + neg_ref), summed into lsum.
    auto chunk_w = [&](const uint32_t(&cur)[32], uint64_t refx2, uint64_t(&lsum)[4], uint32_t(&pk)[16]) {
        const uint64_t sl2x2 = f2pack(sl2, sl2);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const uint64_t z = f2fma(f2pack(__uint_as_float(cur[2 * c]), __uint_as_float(cur[2 * c + 1])),
                                     sl2x2, refx2);
            float z0, z1;
            f2unpack(z, z0, z1);
            const float p0 = ex2(z0), p1 = ex2(z1);
            lsum[c & 3] = f2add(lsum[c & 3], f2pack(p0, p1));
            pk[c] = Elem<T>::pack2(p0, p1);
        }
    };
    auto chunk_max = [&](const uint32_t(&cur)[32]) -> float {
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 32; c += 8)
#pragma unroll
            for (int a = 0; a < 4; ++a)
                m4[a] = max3(m4[a], __uint_as_float(cur[c + a]), __uint_as_float(cur[c + 4 + a]));
        return fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
    };
    auto lsum_total = [&](const uint64_t(&lsum)[4]) -> float {
        float a0, a1, b0f, b1f, c0f, c1f, d0, d1;
        f2unpack(lsum[0], a0, a1);
        f2unpack(lsum[1], b0f, b1f);
        f2unpack(lsum[2], c0f, c1f);
        f2unpack(lsum[3], d0, d1);
        return ((a0 + a1) + (b0f + b1f)) + ((c0f + c1f) + (d0 + d1));
    };
    // O holds PV of the tiles before this one, complete (the S commit
    // covers it): scale the rows whose reference moved
    auto rescale_o = [&](float a) {
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t ov[32];
            tc05::tmem_ld32(to + cc * 32, ov);
            tc05::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * a);
            tc05::tmem_st32(to + cc * 32, ov);
        }
    };
    static_assert(N == 128, "four 32-key chunks per tile");
    // P chunk c lands on S columns 16c .. 16c+15, so storing P chunks 0-3
    // overwrites S chunks 0 and 1 only; S chunks 2 and 3 stay intact.
    float l_add = 0.f, alpha = 1.f;
    bool full = !__all_sync(kAll, m_ref != -INFINITY);
    if (full && __all_sync(kAll, m_ref == -INFINITY)) {
        // every row's first tile: the reference starts at the largest of its
        // first 8 logits, and the sweep below raises it where needed (a
        // causal or context-end mask hides a suffix of the keys, so a row
        // that sees none of these sees nothing in the tile and keeps -inf)
        uint32_t v8[8];
        tc05::tmem_ld8(ts, v8);
        tc05::tmem_wait_ld();
        float m8 = -INFINITY;
#pragma unroll
        for (int c = 0; c < 8; ++c)
            if (key0 + c <= pos) m8 = fmaxf(m8, __uint_as_float(v8[c]));
        m_ref = m8 * sl2;                           // the scale is positive
        full = !__all_sync(kAll, m_ref != -INFINITY);
    }
    if (!full) {
        // Most tiles keep every row's reference: one sweep at it.  The P
        // of chunks 0 and 1 is held until no row of the warp has a logit
        // more than 8 above its reference there (else the tile is redone
        // from the intact S); chunks 2 and 3 are stored at once and
        // checked after, their S still intact for a recomputation.
        const uint64_t refx2 = f2pack(-m_ref, -m_ref);
        uint64_t lA[4] = {0, 0, 0, 0}, lB[4] = {0, 0, 0, 0};
        uint32_t b0[32], b1[32], pk0[16], pk1[16];
        tc05::tmem_ld32(ts, b0);
        tc05::tmem_ld32(ts + 32, b1);
        tc05::tmem_wait_ld();
        mask(b0, 0);
        mask(b1, 32);
        const float cmA = fmaxf(chunk_max(b0), chunk_max(b1));
        chunk_w(b0, refx2, lA, pk0);
        chunk_w(b1, refx2, lA, pk1);
        tc05::tmem_ld32(ts + 64, b0);
        tc05::tmem_ld32(ts + 96, b1);
        if (__any_sync(kAll, cmA * sl2 - m_ref > 8.f)) {
            tc05::tmem_wait_ld();
            full = true;                            // nothing stored: redo from S
        } else {
            tc05::tmem_st16(ts, pk0);
            tc05::tmem_st16(ts + 16, pk1);
            tc05::tmem_wait_ld();
            mask(b0, 64);
            mask(b1, 96);
            const float cmB = fmaxf(chunk_max(b0), chunk_max(b1));
            chunk_w(b0, refx2, lB, pk0);
            tc05::tmem_st16(ts + 32, pk0);
            chunk_w(b1, refx2, lB, pk1);
            tc05::tmem_st16(ts + 48, pk1);
            if (!__any_sync(kAll, cmB * sl2 - m_ref > 8.f)) {
                l_add = lsum_total(lA) + lsum_total(lB);
            } else {
                // a logit of chunk 2 or 3 rose more than 8 above its row's
                // reference: move to the row maximum, rescale the P of
                // chunks 0 and 1 and O, recompute chunks 2 and 3
                const float mt = fmaxf(cmA, cmB) * sl2;
                const bool raise = mt > m_ref + 8.f;
                const float new_ref = raise ? mt : m_ref;
                alpha = raise ? ex2(m_ref - new_ref) : 1.f;
                m_ref = new_ref;
                tc05::tmem_wait_st();
                if (__any_sync(kAll, alpha != 1.f)) {
#pragma unroll
                    for (int ch = 0; ch < 2; ++ch) {
                        uint32_t pv16[16];
                        tc05::tmem_ld16(ts + 16 * ch, pv16);
                        tc05::tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            float lo, hi;
                            Elem<T>::widen2(pv16[e], lo, hi);
                            pv16[e] = Elem<T>::pack2(lo * alpha, hi * alpha);
                        }
                        tc05::tmem_st16(ts + 16 * ch, pv16);
                    }
                    if (o_valid) rescale_o(alpha);
                }
                const uint64_t ref2 = f2pack(-m_ref, -m_ref);
                uint64_t lC[4] = {0, 0, 0, 0};
                chunk_w(b0, ref2, lC, pk0);
                tc05::tmem_st16(ts + 32, pk0);
                chunk_w(b1, ref2, lC, pk1);
                tc05::tmem_st16(ts + 48, pk1);
                l_add = lsum_total(lA) * alpha + lsum_total(lC);
            }
        }
    }
    if (full) {
        // rows that have seen only masked keys, or a jump in chunk 0 or 1:
        // the row maximum first
        float mx = -INFINITY;
#pragma unroll
        for (int hh = 0; hh < N / 64; ++hh) {
            uint32_t va[32], vb[32];
            tc05::tmem_ld32(ts + 64 * hh, va);
            tc05::tmem_ld32(ts + 64 * hh + 32, vb);
            tc05::tmem_wait_ld();
            mask(va, 64 * hh);
            mask(vb, 64 * hh + 32);
            mx = fmaxf(mx, fmaxf(chunk_max(va), chunk_max(vb)));
        }
        const float mt = mx * sl2;                  // the scale is positive
        const bool raise = mt > m_ref + 8.f;
        const float new_ref = raise ? mt : m_ref;
        alpha = (raise && m_ref != -INFINITY) ? ex2(m_ref - new_ref) : 1.f;
        m_ref = new_ref;
        if (o_valid && __any_sync(kAll, alpha != 1.f)) rescale_o(alpha);
        // weights at the new reference, the next chunk's load overlapping
        // this chunk's arithmetic (P chunk c lands on S columns already read)
        const float nr = new_ref == -INFINITY ? 0.f : -new_ref;   // rows that see nothing yet
        const uint64_t refx2 = f2pack(nr, nr);
        uint64_t lsum[4] = {0, 0, 0, 0};
        uint32_t buf[2][32];
        tc05::tmem_ld32(ts, buf[0]);
        tc05::tmem_wait_ld();
#pragma unroll
        for (int ch = 0; ch < N / 32; ++ch) {
            uint32_t(&cur)[32] = buf[ch & 1];
            if (ch + 1 < N / 32) tc05::tmem_ld32(ts + 32 * (ch + 1), buf[(ch + 1) & 1]);
            mask(cur, 32 * ch);
            uint32_t pk[16];
            chunk_w(cur, refx2, lsum, pk);
            tc05::tmem_st16(ts + 16 * ch, pk);
            tc05::tmem_wait_ld();
        }
        l_add = lsum_total(lsum);
    }
    l = l * alpha + l_add;
}

}  // namespace tcsm
}  // namespace pkv
