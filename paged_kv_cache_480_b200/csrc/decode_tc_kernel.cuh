// Split-context decode attention on the sm_100a tensor cores for groups of
// many query heads per KV head (GQA with large groups, MQA).
//
// One decode step: every sequence s has one query token at position L - 1
// (L = context_lens[s]) attending to all L keys of its blocks ("Efficient
// Memory Management for Large Language Model Serving with PagedAttention"
// summary page, section 2: the kernel fetches K/V block by block through the
// block table).  With G query heads sharing a KV head, the G rows of q against
// one K/V tile are a dense product (G * 4 * head_size flops per 2 * head_size
// * elem bytes of K/V), large enough to need the tensor cores once G reaches
// about 16.
//
// Work: a unit is (sequence s, KV head g, slice of up to 128 of its query
// heads); its keys form ceil(L / 128) tiles of N = 128 keys.  The tiles of all
// units, in order, are split into contiguous ranges of equal cost, one per CTA
// of a grid of kDecodeTcCtas persistent CTAs (one per SM); a unit costs its
// tiles plus kTcUnitCost for its start and its partial write.  A CTA streams
// its range without a break at unit boundaries: the K/V rings and the
// tensor-core pipeline run on across units, q is double-buffered per unit.
//
// Rows of the M = 128 tile are the unit's heads (rows past them hold zeros and
// are never written out).  The CTA's tiles alternate between two halves x =
// tile % 2; each half keeps its own S_x, O_x in tensor memory and its own
// softmax warpgroup, so the tensor core runs one half's products while the
// other half's softmax works (issue order QK(i), PV(i-1), QK(i+1), PV(i)).
// For every unit it touches, each half writes its unnormalised O, reference
// maximum and weight sum as one partial result, in slot 2 * (cta + unit) + x
// (disjoint between units because consecutive units share at most one CTA);
// the log-sum-exp merge kernel (merge_kernel.cuh) combines a unit's partials.
// Roles:
//   warps 0-3, 4-7  softmax and partial write of half 0 and 1, one row per thread;
//   warp 8          issues the MMAs (one thread);
//   warp 9          streams q and K by TMA;  warp 10  streams V by TMA and
//                   zeroes the V rows past a context's end in its last block.
// Every wait is bounded; the tensor memory is freed on every path.
#pragma once

#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "tc05.cuh"
#include "tc_softmax.cuh"

namespace pkv {

// CTAs of the tensor-core decode: one per SM of a B200.  The work split and
// the partial-result layout depend on it, not on the device the call runs on.
constexpr int kDecodeTcCtas = 148;
// The cost of a unit's start and partial write in key tiles (measured: a CTA
// whose range meets two units ends about two tiles' time later than one
// whose range meets one).
constexpr int kTcUnitCost = 2;

struct DecodeTcParams {
    float* part_acc;                  // [2 * (ctas + units)][rows][D] unnormalised O
    float2* part_ml;                  // [2 * (ctas + units)][rows] (m_ref in log2 units, l)
    int32_t* prefix;                  // [S + 1] cost of one unit of each earlier sequence, summed (CTA 0 writes)
    const int32_t* block_tables;      // [S][MB]
    const int32_t* context_lens;      // [S]
    unsigned int* errors;
    float scale_log2;                 // softmax scale * log2(e)
    int num_seqs, num_heads, num_kv_heads, num_blocks, max_blocks_per_seq;
    int max_len;                      // lengths above it (or negative) count as 0 and are flagged
    int group;                        // G = num_heads / num_kv_heads
    int slices;                       // ceil(G / 128) units per KV head
    int rows;                         // min(G, 128): rows of a partial slot and of the q box
    int cache_rows;                   // rows of the [NB * Hkv * bs][D] view of a cache
    uint32_t wait_limit;              // polls before a wait for progress gives up
};

#ifndef PKV_DECODE_TC_KST128
#define PKV_DECODE_TC_KST128 3
#endif
#ifndef PKV_DECODE_TC_VST128
#define PKV_DECODE_TC_VST128 2
#endif

template <typename T, int D, int BS>
struct DecodeTcShape {
    static constexpr int M = 128;               // rows (query heads) per tile
    static constexpr int N = 128;               // keys per tile
    static constexpr int DH = D / 64;           // 64-dim halves (one 128-byte swizzle row each)
    static constexpr int BPT = N / BS;          // cache blocks per key tile
    static constexpr int KST = D == 64 ? 5 : PKV_DECODE_TC_KST128;   // K stages
    static constexpr int VST = D == 64 ? 4 : PKV_DECODE_TC_VST128;   // V stages
    static constexpr uint32_t Q_HALF = M * 128;
    static constexpr uint32_t KV_HALF = N * 128;
    static constexpr uint32_t Q_BYTES = DH * Q_HALF;         // one q buffer
    static constexpr uint32_t KV_BYTES = DH * KV_HALF;       // K or V of one key tile
    static constexpr uint32_t OFF_K = 2 * Q_BYTES;
    static constexpr uint32_t OFF_V = OFF_K + KST * KV_BYTES;
    static constexpr uint32_t OFF_BAR = OFF_V + VST * KV_BYTES;
    static constexpr uint32_t SMEM = OFF_BAR + 512 + 1024;  // barriers, scratch, 1 KB alignment slack
    static constexpr uint32_t TM_TILE = 256;                // columns per half
    static constexpr uint32_t TM_S = 0;                     // S (N fp32 columns); P over its first N/2
    static constexpr uint32_t TM_O = N;                     // O at columns N .. N + D
    static constexpr uint32_t TM_COLS = 512;
    static_assert(N + D <= (int)TM_TILE, "tensor-memory budget");
    static_assert(N % BS == 0, "key tile holds whole blocks");
    static_assert(8 * (14 + 2 * (KST + VST)) <= 256, "barrier area");
    static_assert(SMEM <= 232448, "shared memory per CTA");
};

constexpr uint32_t kDecodeTcThreads = 352;

// Key tiles of one unit of sequence s (0 for an empty or invalid length).
__device__ __forceinline__ int tc_seq_len(const DecodeTcParams& p, int s) {
    const int L = __ldg(p.context_lens + s);
    return (L < 0 || L > p.max_len) ? 0 : L;
}

// Walk over the segments of a CTA's range: maximal runs of consecutive tiles
// of one unit.  Every role walks the same sequence independently.  Costs are
// counted in the range's own units: the unit's kTcUnitCost, then its tiles.
struct TcSegWalk {
    int s, u, t;       // sequence, unit within the sequence, next tile of that unit
    int L, Ts;         // the sequence's length and tiles per unit
    int left;          // cost from the unit's first tile to the end of the CTA's range
    int NU;            // units per sequence
    // Next segment: unit (s, u), tiles [t0, t0 + n).  False at the range's end.
    __device__ __forceinline__ bool next(const DecodeTcParams& p, int& ss, int& uu, int& t0, int& n, int& LL,
                                         int& TT) {
        while (t >= Ts) {                           // unit done (or empty): the next one
            if (Ts > 0) left -= Ts + kTcUnitCost;
            t = 0;
            if (++u == NU) {
                u = 0;
                if (++s >= p.num_seqs) return false;
                L = tc_seq_len(p, s);
                Ts = (L + 127) / 128;
            }
        }
        if (t >= left) return false;
        n = min(Ts - t, left - t);
        ss = s;
        uu = u;
        t0 = t;
        LL = L;
        TT = Ts;
        t += n;
        return true;
    }
};

template <typename T, int D, int BS>
__global__ void __launch_bounds__(kDecodeTcThreads, 1)
    paged_decode_tc_kernel(const DecodeTcParams p, const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
    using S = DecodeTcShape<T, D, BS>;
    using namespace tcsm;
    constexpr int KST = S::KST, VST = S::VST;
    constexpr int N = S::N;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw_s = smem_addr(smem_raw);
    const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
    unsigned char* smem = smem_raw + pad;
    const uint32_t sm = raw_s + pad;                // 1024-byte aligned shared address
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nthreads = blockDim.x, nwarps = nthreads >> 5;
    const uint32_t wl = p.wait_limit;
    const int G = p.group, GR = p.rows, NU = p.num_kv_heads * p.slices;
    const int C = gridDim.x, c = blockIdx.x;

    // ---- barriers, tensor memory, scratch ----
    const uint32_t bar = sm + S::OFF_BAR;
    auto bar_qfull = [&](int b) { return bar + 8 * b; };
    auto bar_qempty = [&](int b) { return bar + 8 * (2 + b); };
    auto bar_kfull = [&](int st) { return bar + 8 * (4 + st); };
    auto bar_kempty = [&](int st) { return bar + 8 * (4 + KST + st); };
    auto bar_vfull = [&](int st) { return bar + 8 * (4 + 2 * KST + st); };
    auto bar_vempty = [&](int st) { return bar + 8 * (4 + 2 * KST + VST + st); };
    constexpr int B0 = 4 + 2 * KST + 2 * VST;
    auto bar_s = [&](int x) { return bar + 8 * (B0 + x); };        // QK into S_x done (and all before it)
    auto bar_p = [&](int x) { return bar + 8 * (B0 + 2 + x); };    // P_x written (128 arrivals)
    auto bar_o = [&](int x) { return bar + 8 * (B0 + 4 + x); };    // a unit's last PV into O_x done
    auto bar_ofree = [&](int x) { return bar + 8 * (B0 + 6 + x); };  // O_x read out (128 arrivals)
    const uint32_t bar_vz = bar + 8 * (B0 + 8);
    const uint32_t bar_fin = bar + 8 * (B0 + 9);
    uint32_t* tm_holder = reinterpret_cast<uint32_t*>(smem + S::OFF_BAR + 256);
    int* scratch = reinterpret_cast<int*>(smem + S::OFF_BAR + 320);   // [0..15] warp sums, [16..19] start
    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_qfull(b), 1);
            mbar_init(bar_qempty(b), 1);
        }
        for (int st = 0; st < KST; ++st) {
            mbar_init(bar_kfull(st), 1);
            mbar_init(bar_kempty(st), 1);
        }
        for (int st = 0; st < VST; ++st) {
            mbar_init(bar_vfull(st), 1);
            mbar_init(bar_vempty(st), 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(bar_s(x), 1);
            mbar_init(bar_p(x), 128);
            mbar_init(bar_o(x), 1);
            mbar_init(bar_ofree(x), 128);
        }
        mbar_init(bar_vz, 1);
        mbar_init(bar_fin, 1);
        fence_mbar_init();
    }
    if (threadIdx.x == 32) {
        tc05::prefetch_tmap(&tm_q);
        tc05::prefetch_tmap(&tm_k);
        tc05::prefetch_tmap(&tm_v);
    }
    if (warp == 0) {
        tc05::tmem_alloc(smem_addr(tm_holder), S::TM_COLS);
        tc05::tmem_relinquish();
    }
    // rows of both q buffers past the unit's heads stay zero (the q box never
    // writes them; zeros keep their softmax finite and off the redo path)
    if (GR < S::M) {
        const int nz = (S::M - GR) * 8;                 // 16-byte chunks per 64-dim half
        for (int i = threadIdx.x; i < 2 * S::DH * nz; i += nthreads) {
            const int h = i / nz, k = i - h * nz;       // h = buffer * DH + dh
            *reinterpret_cast<uint4*>(smem + h * S::Q_HALF + GR * 128 + k * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async();   // visible to the tensor core's reads of q
    }

    griddep_wait();
    griddep_launch();                               // the merge kernel may get resident; it waits for us

    // ---- the CTA's range: [floor(c V / C), floor((c + 1) V / C)) of the cost
    // index, V = NU * sum_s w(s), w(s) = kTcUnitCost + tiles(s) for a sequence
    // with keys, else 0; the unit (s, u) spans [NU W(s) + u w(s), + w(s)) with
    // W(s) = sum of w over earlier sequences, its tiles the last tiles(s) of it.
    // CTA 0 also publishes W for the merge.
    auto block_sum = [&](int v) -> int {            // all threads; returns the block total
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(kAll, v, off);
        if (lane == 0) scratch[warp] = v;
        __syncthreads();
        int tot = 0;
        for (int w = 0; w < nwarps; ++w) tot += scratch[w];
        __syncthreads();
        return tot;
    };
    // the block tables to L2 while the lengths are summed (a slice per CTA)
    if (warp == 10) {
        const uint32_t lines = (uint32_t)(((int64_t)p.num_seqs * p.max_blocks_per_seq + 31) / 32);
        const uint32_t per = (lines + C - 1) / C, hi = min(lines, (uint32_t)(c + 1) * per);
        for (uint32_t i = (uint32_t)c * per + lane; i < hi; i += 32)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(p.block_tables + (size_t)i * 32));
    }
    // a sequence's cost w(s); c == 0 flags lengths out of range
    auto seq_cost = [&](int s) -> int {
        if (s >= p.num_seqs) return 0;
        const int raw = __ldg(p.context_lens + s);
        const int L = tc_seq_len(p, s);
        if (c == 0 && L != raw) flag_error(p.errors, PKV_DEVERR_CONTEXT);
        return L > 0 ? (L + 127) / 128 + kTcUnitCost : 0;
    };
    // the CTA whose range holds cost index v0 in sequence s (prefix pre, cost w) notes it
    auto note_start = [&](int s, int64_t pre, int w, int64_t v0) {
        if (w > 0 && pre * NU <= v0 && v0 < (pre + w) * NU) {
            scratch[16] = s;
            scratch[17] = (int)(v0 - pre * NU);         // offset of the start in s's units
            scratch[18] = (int)pre;
        }
    };
    int64_t v0, v1;
    if (p.num_seqs <= nthreads) {
        // one chunk: a single block scan gives every prefix and the total
        const int s = threadIdx.x;
        const int w = seq_cost(s);
        int incl = w;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(kAll, incl, off);
            if (lane >= off) incl += v;
        }
        if (lane == 31) scratch[warp] = incl;
        if (threadIdx.x == 0) scratch[16] = -1;
        __syncthreads();
        int before = 0, all = 0;
        for (int wp = 0; wp < nwarps; ++wp) {
            if (wp < warp) before += scratch[wp];
            all += scratch[wp];
        }
        const int64_t vtot = (int64_t)all * NU;
        v0 = vtot * c / C;
        v1 = vtot * (c + 1) / C;
        const int64_t pre = before + incl - w;    // W(s)
        if (s < p.num_seqs) {
            if (c == 0) p.prefix[s] = (int32_t)pre;
            note_start(s, pre, w, v0);
        }
        if (c == 0 && threadIdx.x == 0) p.prefix[p.num_seqs] = all;
    } else {
        // pass 1: V; pass 2: the prefixes and the sequence holding the start
        int64_t total = 0;
        for (int base = 0; base < p.num_seqs; base += nthreads) total += block_sum(seq_cost(base + threadIdx.x));
        const int64_t vtot = total * NU;
        v0 = vtot * c / C;
        v1 = vtot * (c + 1) / C;
        if (threadIdx.x == 0) scratch[16] = -1;
        __syncthreads();
        int64_t carry = 0;
        for (int base = 0; base < p.num_seqs; base += nthreads) {
            const int s = base + threadIdx.x;
            const int w = s < p.num_seqs && tc_seq_len(p, s) > 0 ? (tc_seq_len(p, s) + 127) / 128 + kTcUnitCost : 0;
            int incl = w;                           // inclusive scan over the block
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_up_sync(kAll, incl, off);
                if (lane >= off) incl += v;
            }
            if (lane == 31) scratch[warp] = incl;
            __syncthreads();
            int before = 0, chunk = 0;
            for (int wp = 0; wp < nwarps; ++wp) {
                if (wp < warp) before += scratch[wp];
                chunk += scratch[wp];
            }
            const int64_t pre = carry + before + incl - w;    // W(s)
            if (s < p.num_seqs) {
                if (c == 0) p.prefix[s] = (int32_t)pre;
                note_start(s, pre, w, v0);
            }
            carry += chunk;
            const bool found = __syncthreads_or(scratch[16] >= 0);
            if (found && c != 0) break;
        }
        if (c == 0 && threadIdx.x == 0) p.prefix[p.num_seqs] = (int32_t)carry;
    }
    __syncthreads();
    TcSegWalk walk0;
    walk0.NU = NU;
    bool has_work = false;
    if (v1 > v0 && scratch[16] >= 0) {
        walk0.s = scratch[16];
        walk0.L = tc_seq_len(p, walk0.s);
        walk0.Ts = (walk0.L + 127) / 128;
        const int w = walk0.Ts + kTcUnitCost, o = scratch[17];
        walk0.u = o / w;
        walk0.t = max(0, o - walk0.u * w - kTcUnitCost);
        // the range ends at most one range length past the unit's first tile
        walk0.left = (int)(v1 - ((int64_t)scratch[18] * NU + (int64_t)walk0.u * w + kTcUnitCost));
        has_work = walk0.t < walk0.left;
    } else {
        walk0.s = walk0.u = walk0.t = walk0.L = walk0.Ts = walk0.left = 0;
    }
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    const uint32_t tm = *tm_holder;

    auto q_base = [&](int b) { return sm + (uint32_t)b * S::Q_BYTES; };
    auto k_base = [&](int st) { return sm + S::OFF_K + (uint32_t)st * S::KV_BYTES; };
    auto v_base = [&](int st) { return sm + S::OFF_V + (uint32_t)st * S::KV_BYTES; };

    if (!has_work) {
        // no tile in the range (more CTAs than work): nothing to do
    } else if (warp >= 9) {
        // ===================== TMA producers: warp 9 q and K, warp 10 V =====================
        const bool is_v = warp == 10;
        const int nst = is_v ? VST : KST;
        const CUtensorMap* map = is_v ? &tm_v : &tm_k;
        TcSegWalk w = walk0;
        int jt = 0, js = 0, qloads[2] = {0, 0};
        bool ok = true;
        // V rows of the pending tile past its context end, zeroed once it lands
        int vz_jt = -1, vz_r0 = 0, vz_r1 = 0;
        auto do_vz = [&]() {
            const int st = vz_jt % VST;
            if (warp_wait(bar_vfull(st), (vz_jt / VST) & 1, wl)) {
                const int rows = vz_r1 - vz_r0;
                for (int i = lane; i < rows * S::DH * 8; i += 32) {   // 16-byte chunks
                    const int dh = i / (rows * 8);
                    const int rem = i - dh * rows * 8;
                    *reinterpret_cast<uint4*>(smem + (v_base(st) - sm) + dh * S::KV_HALF + (vz_r0 + rem / 8) * 128 +
                                              (rem % 8) * 16) = make_uint4(0u, 0u, 0u, 0u);
                }
                fence_proxy_async();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_vz);
            } else {
                ok = false;
            }
            vz_jt = -1;
        };
        int s, u, t0, n, L, Ts;
        while (ok && w.next(p, s, u, t0, n, L, Ts)) {
            const int g = u / p.slices, sl = u - g * p.slices;
            if (!is_v) {
                // q of the unit into buffer js % 2, once the QKs of unit js - 2 are done
                const int b = js & 1;
                if (js >= 2 && !warp_wait(bar_qempty(b), ((js >> 1) - 1) & 1, wl)) { ok = false; break; }
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar_qfull(b), (uint32_t)(S::DH * GR * 128));
                    for (int dh = 0; dh < S::DH; ++dh)
                        tc05::tma_load_3d(q_base(b) + dh * S::Q_HALF, &tm_q, dh * 64, g * G + sl * S::M, s,
                                          bar_qfull(b));
                }
                ++qloads[b];
            }
            const int nblk = (L + BS - 1) / BS;
            // cache row of block `lane` of the segment's tile i (one coalesced load
            // per tile, a tile ahead of its copies); past the sequence's blocks, or
            // for a bad id, the row past the pool, which TMA fills with zeros
            auto tile_row = [&](int i) -> int {
                int row = p.cache_rows;
                const int lb = (t0 + i) * S::BPT + lane;
                if (lane < S::BPT && lb < nblk) {
                    const int phys = __ldg(p.block_tables + (size_t)s * p.max_blocks_per_seq + lb);
                    if (phys >= 0 && phys < p.num_blocks) row = (phys * p.num_kv_heads + g) * BS;
                    else if (!is_v) flag_error(p.errors, PKV_DEVERR_BLOCK_ID);
                }
                return row;
            };
            int next_row = tile_row(0);
            for (int i = 0; i < n; ++i, ++jt) {
                const int cur_row = next_row;
                if (i + 1 < n) next_row = tile_row(i + 1);
                const int st = jt % nst;
                // the pending zeroing must happen before its stage is waited for again
                if (is_v && vz_jt >= 0 && jt >= vz_jt + VST) do_vz();
                if (jt >= nst && !warp_wait(is_v ? bar_vempty(st) : bar_kempty(st), ((jt / nst) - 1) & 1, wl)) {
                    ok = false;
                    break;
                }
                const uint32_t full = is_v ? bar_vfull(st) : bar_kfull(st);
                const uint32_t dst = is_v ? v_base(st) : k_base(st);
                if (lane == 0) mbar_arrive_expect_tx(full, S::KV_BYTES);
#pragma unroll
                for (int bi = 0; bi < S::BPT; ++bi) {
                    const int row = __shfl_sync(kAll, cur_row, bi);
                    if (lane == 0)
                        for (int dh = 0; dh < S::DH; ++dh)
                            tc05::tma_load_2d(dst + dh * S::KV_HALF + bi * BS * 128, map, dh * 64, row, full);
                }
                if (is_v && t0 + i == Ts - 1) {
                    // the unit's last tile: V rows from the context end to the end of
                    // its last block hold whatever the pool holds there
                    const int r0 = L - (Ts - 1) * N;
                    const int r1 = min(nblk * BS - (Ts - 1) * N, N);
                    if (r0 < r1) {
                        if (vz_jt >= 0) do_vz();
                        vz_jt = jt;
                        vz_r0 = r0;
                        vz_r1 = r1;
                    }
                }
            }
            ++js;
        }
        if (is_v && vz_jt >= 0 && ok) do_vz();
        if (!ok && lane == 0) flag_error(p.errors, PKV_DEVERR_WAIT);
        if (lane == 0) {
            // every copy requested above lands before this warp leaves (the last
            // copy into each stage and each q buffer; earlier ones were consumed
            // before their buffer was refilled)
            for (int b = 0; b < 2; ++b)
                if (qloads[b] > 0) mbar_wait_bounded(bar_qfull(b), (qloads[b] - 1) & 1, kWaitLimit);
            for (int t = max(0, jt - nst); t < jt; ++t)
                mbar_wait_bounded(is_v ? bar_vfull(t % nst) : bar_kfull(t % nst), (t / nst) & 1, kWaitLimit);
        }
        __syncwarp();
    } else if (warp == 8) {
        // ===================== MMA issue =====================
        if (lane == 0) {
            constexpr uint32_t idesc_qk = tc05::instr_desc(kBf16, 128, N, false, false);
            constexpr uint32_t idesc_pv = tc05::instr_desc(kBf16, 128, D, false, true);
            // operand descriptors of q buffer 0 and stage 0; the start-address
            // field (bits 0-13, address / 16) is advanced by plain addition
            const uint64_t dq = tc05::smem_desc(q_base(0), 16, 1024);
            const uint64_t dk = tc05::smem_desc(k_base(0), 16, 1024);
            const uint64_t dv = tc05::smem_desc(v_base(0), S::KV_HALF, 1024);
            TcSegWalk w = walk0;
            bool ok = true;
            int jt = 0, js = 0, vzc = 0;
            int px[2] = {0, 0};                          // P_x phases consumed
            int ox[2] = {0, 0};                          // units whose O_x accumulation began
            struct Pend { int jt, x, first, last, vz; } prev = {-1, 0, 0, 0, 0};
            auto pv = [&](const Pend& e) -> bool {       // O_x += P_x V_jt
                const int sv = e.jt % VST;
                if (!mbar_wait_bounded(bar_vfull(sv), (e.jt / VST) & 1, wl)) return false;
                if (e.vz) {
                    if (!mbar_wait_bounded(bar_vz, vzc & 1, wl)) return false;
                    ++vzc;
                }
                if (!mbar_wait_bounded(bar_p(e.x), px[e.x] & 1, wl)) return false;
                ++px[e.x];
                if (e.first) {
                    // the half's previous unit must be read out before O_x restarts
                    if (ox[e.x] >= 1 && !mbar_wait_bounded(bar_ofree(e.x), (ox[e.x] - 1) & 1, wl)) return false;
                    ++ox[e.x];
                }
                tc05::fence_after_sync();
                const uint32_t base = tm + e.x * S::TM_TILE;
                const uint64_t vd = dv + (uint64_t)((sv * S::KV_BYTES) >> 4);
                // k-th 16 keys: 16 rows of 128 bytes further; P pairs 8 columns further
#pragma unroll
                for (int k = 0; k < N / 16; ++k)
                    tc05::mma_ts(base + S::TM_O, base + S::TM_S + 8 * k, vd + (uint64_t)(k * 128), idesc_pv,
                                 (!e.first || k > 0) ? 1u : 0u);
                tc05::commit(bar_vempty(sv));
                if (e.last) tc05::commit(bar_o(e.x));
                return true;
            };
            int s, u, t0, n, L, Ts;
            while (ok && w.next(p, s, u, t0, n, L, Ts)) {
                const int b = js & 1;
                if (!mbar_wait_bounded(bar_qfull(b), (js >> 1) & 1, wl)) { ok = false; break; }
                const int nblk = (L + BS - 1) / BS;
                const bool unit_vz = t0 + n == Ts && L - (Ts - 1) * N < min(nblk * BS - (Ts - 1) * N, N);
                for (int i = 0; i < n; ++i, ++jt) {
                    const int x = jt & 1;
                    if (!mbar_wait_bounded(bar_kfull(jt % KST), (jt / KST) & 1, wl)) { ok = false; break; }
                    tc05::fence_after_sync();
                    {                                    // S_x = q K_jt^T
                        const uint32_t d = tm + x * S::TM_TILE + S::TM_S;
                        const uint64_t ad = dq + (uint64_t)((b * S::Q_BYTES) >> 4);
                        const uint64_t bd = dk + (uint64_t)(((jt % KST) * S::KV_BYTES) >> 4);
                        // k-th 16-wide slice: +32 bytes inside a swizzle row, next half after 4
#pragma unroll
                        for (int k = 0; k < D / 16; ++k) {
                            const uint32_t qoff = ((k >> 2) * S::Q_HALF + (k & 3) * 32) >> 4;
                            const uint32_t koff = ((k >> 2) * S::KV_HALF + (k & 3) * 32) >> 4;
                            tc05::mma_ss(d, ad + qoff, bd + koff, idesc_qk, k > 0 ? 1u : 0u);
                        }
                    }
                    tc05::commit(bar_s(x));
                    tc05::commit(bar_kempty(jt % KST));
                    if (i == n - 1) tc05::commit(bar_qempty(b));
                    if (prev.jt >= 0 && !pv(prev)) { ok = false; break; }
                    // this tile's half: its first tile of the unit are i = 0, 1, its last i = n-2, n-1
                    prev = {jt, x, i < 2 ? 1 : 0, i >= n - 2 ? 1 : 0, (unit_vz && i == n - 1) ? 1 : 0};
                }
                ++js;
            }
            if (ok && prev.jt >= 0 && !pv(prev)) ok = false;
            if (!ok) flag_error(p.errors, PKV_DEVERR_WAIT);
            // every MMA issued above is complete before the tensor memory is freed
            tc05::commit(bar_fin);
            mbar_wait_bounded(bar_fin, 0, kWaitLimit);
        }
    } else {
        // ===================== softmax and partials: one row (query head) per thread =====================
        const int x = warp >> 2;                        // half
        const int wq = warp & 3;
        const int r = wq * 32 + lane;                   // row = query head (slice start) + r
        const uint32_t trow = tm + x * S::TM_TILE + ((uint32_t)(wq * 32) << 16);
        const float sl2 = p.scale_log2;
        TcSegWalk w = walk0;
        bool ok = true;
        int jt = 0, nx = 0, ox = 0;                     // tile counter; S_x phases; units of this half
        int s, u, t0, n, L, Ts;
        while (w.next(p, s, u, t0, n, L, Ts)) {
            const int sl = u % p.slices;
            const bool valid = r < min(S::M, G - sl * S::M);
            // partial slot of this half for the unit: 2 * (cta + unit) + x
            const size_t prow = (2 * ((size_t)c + (size_t)s * NU + u) + x) * GR + r;
            const int i0 = ((jt & 1) == x) ? 0 : 1;     // this half's first tile of the segment
            const int cnt = n > i0 ? (n - i0 + 1) / 2 : 0;
            jt += n;
            if (!ok || cnt == 0) {
                if (valid) p.part_ml[prow] = make_float2(-INFINITY, 0.f);
                continue;
            }
            float m_ref = -INFINITY, l = 0.f;           // reference max (log2 units), sum of weights
            // every row sees keys 0 .. L - 1 (rows past the heads too: the same
            // mask keeps their logits finite past the context end)
            for (int k = 0; k < cnt; ++k) {
                if (!warp_wait(bar_s(x), nx & 1, wl)) { ok = false; break; }
                ++nx;
                tc05::fence_after_sync();
                softmax_tile<T, D>(trow + S::TM_S, trow + S::TM_O, (t0 + i0 + 2 * k) * N, L - 1, sl2, k > 0, m_ref, l);
                tc05::tmem_wait_st();
                tc05::fence_before_sync();
                mbar_arrive(bar_p(x));
            }
            // ---- the unnormalised O of this half to its partial slot ----
            if (ok && warp_wait(bar_o(x), ox & 1, wl)) {
                tc05::fence_after_sync();
                float4* dst = reinterpret_cast<float4*>(p.part_acc + prow * D);
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t ov[32];
                    tc05::tmem_ld32(trow + S::TM_O + cc * 32, ov);
                    tc05::tmem_wait_ld();
                    if (valid) {
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            dst[cc * 8 + v] = make_float4(__uint_as_float(ov[4 * v]), __uint_as_float(ov[4 * v + 1]),
                                                          __uint_as_float(ov[4 * v + 2]),
                                                          __uint_as_float(ov[4 * v + 3]));
                    }
                }
                tc05::fence_before_sync();
                mbar_arrive(bar_ofree(x));
            } else {
                ok = false;
            }
            ++ox;
            if (valid) p.part_ml[prow] = ok ? make_float2(m_ref, l) : make_float2(-INFINITY, 0.f);
        }
        if (!ok && lane == 0) flag_error(p.errors, PKV_DEVERR_WAIT);
    }
    tc05::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc05::fence_after_sync();
        tc05::tmem_dealloc(tm, S::TM_COLS);
    }
}

}  // namespace pkv
