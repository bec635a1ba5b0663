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
// CTA share each K/V tile brought into shared memory.  A query tile holds
// QT = floor(128 / G) queries; when G does not divide 128 its last
// 128 - QT * G rows are zero and never written out.  Roles:
//   warps 0-3 and 4-7  softmax of query tile 0 and 1, one row per thread
//                      (warp w reaches tensor-memory lanes 32(w%4) .. +31);
//   warp 8             issues the MMAs (one thread);
//   warps 9 and 10     stream K and V tiles through two rings of stages
//                      with TMA, each refilling a stage once the products
//                      that read it are done.
// Per key tile i of N = 128 keys and query tile x, in tensor memory
// columns [256x, 256x + 256): S_x (128 fp32 columns), P_x over the first 64
// of them (16-bit pairs), O_x (D fp32 columns) after S_x:
//   S_x  = Q_x K_i^T    tcgen05.mma, A = Q and B = K from 128-byte-swizzled
//                       shared memory (K-major);
//   P_x  = exp2(S_x * scale*log2e - m_ref) rounded to the element type;
//   O_x += P_x V_i      tcgen05.mma, A = P from tensor memory, B = V from
//                       shared memory (MN-major).
// The MMA thread issues QK_0(i), PV_1(i-1), QK_1(i), PV_0(i): while one
// softmax warpgroup works on its tile the tensor core runs the other tile's
// two products.  QK_x(i+1) is issued right behind PV_x(i), whose A operand
// P_x it overwrites: tcgen05.mma operations of one thread execute in issue
// order, and a commit covers every earlier operation of its thread, so the
// softmax that sees S_x(i+1) may also rescale O_x.  m_ref is raised (and O
// and l rescaled) only when a row's maximum grows by more than 8 in log2
// units, so O stays exact up to the final division by l.  Masks are applied
// only on tiles that reach past some row's position.  Every wait is
// bounded; the tensor memory is freed on every path.
#pragma once

#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "tc05.cuh"
#include "tc_softmax.cuh"

namespace pkv {

struct PrefillParams {
    void* out;                        // [T][H][D]
    const int32_t* block_tables;      // [S][MB]
    const int32_t* context_lens;      // [S]
    const int32_t* query_start_loc;   // [S + 1]
    unsigned int* errors;
    float scale_log2;                 // softmax scale * log2(e), > 0
    int num_tokens, num_seqs, num_heads, num_kv_heads, num_blocks, max_blocks_per_seq;
    int group;                        // G = num_heads / num_kv_heads, 1 .. 128
    int qt;                           // queries per query tile: floor(128 / G)
    uint32_t wait_limit;              // polls before a wait for progress gives up
    int q_tiles;                      // CTAs (query-tile pairs) per (sequence, KV head)
    int sched_group;                  // (sequence, KV head) pairs per scheduling group, >= 1
    int cache_rows;                   // rows of the [NB * Hkv * bs][D] view of a cache
};

#ifndef PKV_PREFILL_KST128
#define PKV_PREFILL_KST128 3
#endif

#ifndef PKV_PREFILL_VST128
#define PKV_PREFILL_VST128 2
#endif

template <typename T, int D, int BS>
struct PrefillShape {
    static constexpr int M = 128;               // rows per query tile
    static constexpr int N = 128;               // keys per tile
    static constexpr int DH = D / 64;           // 64-dim halves (one 128-byte swizzle row each)
    static constexpr int BPT = N / BS;          // cache blocks per key tile
    static constexpr int KST = D == 64 ? 4 : PKV_PREFILL_KST128;   // K stages
    static constexpr int VST = D == 64 ? 4 : PKV_PREFILL_VST128;   // V stages
    static constexpr uint32_t Q_HALF = M * 128;
    static constexpr uint32_t KV_HALF = N * 128;
    static constexpr uint32_t Q_BYTES = DH * Q_HALF;        // one query tile
    static constexpr uint32_t KV_BYTES = DH * KV_HALF;      // K or V of one key tile
    static constexpr uint32_t OFF_K = 2 * Q_BYTES;
    static constexpr uint32_t OFF_V = OFF_K + KST * KV_BYTES;
    static constexpr uint32_t OFF_BAR = OFF_V + VST * KV_BYTES;
    static constexpr uint32_t SMEM = OFF_BAR + 512 + 1024;  // barriers, TMEM holder, 1 KB alignment slack
    static constexpr uint32_t TM_TILE = 256;                // columns per query tile
    static constexpr uint32_t TM_S = 0;                     // S (N fp32 columns); P over its first N/2
    static constexpr uint32_t TM_O = N;                     // O at columns N .. N + D
    static constexpr uint32_t TM_COLS = 512;
    static_assert(N + D <= (int)TM_TILE, "tensor-memory budget");
    static_assert(N % BS == 0, "key tile holds whole blocks");
    static_assert(8 * (9 + 2 * (KST + VST)) <= 256, "barrier area");
    static_assert(SMEM > 232448 / 2 && SMEM <= 232448, "one CTA per SM");
};

constexpr uint32_t kPrefillThreads = 352;

template <typename T, int D, int BS>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    paged_prefill_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
    using S = PrefillShape<T, D, BS>;
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
    const int G = p.group, QT = p.qt, CQ = 2 * QT;  // heads per KV head; queries per tile and per CTA
    const int QROWS = QT * G;                       // rows of a query tile that hold queries
    const uint32_t wl = p.wait_limit;

    griddep_wait();
    // ---- which queries: the later ones (more keys) are scheduled first ----
    const int Hkv = p.num_kv_heads;
    const int pairs = p.num_seqs * Hkv;
    // groups of p.sched_group (sequence, KV head) pairs, one after the other; inside
    // a group the tiles with most keys go first.  The host sizes groups so
    // that a group's K/V fits in half of L2 while its query tiles read it.
    const int gp = min(p.sched_group, pairs);
    const int per_group = gp * p.q_tiles;
    const int grp = (int)blockIdx.x / per_group;
    const int in_g = (int)blockIdx.x - grp * per_group;
    const int g_pairs = min(gp, pairs - grp * gp);        // the last group may be smaller
    const int tile = p.q_tiles - 1 - in_g / g_pairs;
    const int rest = grp * gp + in_g % g_pairs;
    const int g = rest % Hkv;
    const int s = rest / Hkv;
    const int q0 = p.query_start_loc[s];
    const int n = p.query_start_loc[s + 1] - q0;
    const int L = p.context_lens[s];
    const int i0 = tile * CQ;
    if (n < 0 || n > L || n > p.q_tiles * CQ || L > p.max_blocks_per_seq * BS || q0 < 0 ||
        q0 + n > p.num_tokens) {
        if (threadIdx.x == 0) flag_error(p.errors, PKV_DEVERR_CONTEXT);
        return;
    }
    if (i0 >= n) return;                            // whole CTA, before any barrier or TMEM use
    // key tiles each query tile needs (0: the tile holds no query)
    const int nT0 = (L - n + min(i0 + QT, n) + N - 1) / N;
    const int nT1 = i0 + QT < n ? (L - n + min(i0 + CQ, n) + N - 1) / N : 0;
    auto nTx = [&](int x) { return x ? nT1 : nT0; };
    const bool two = nT1 > 0;
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
    auto bar_kfull = [&](int st) { return bar + 8 * (1 + st); };
    auto bar_kempty = [&](int st) { return bar + 8 * (1 + KST + st); };
    auto bar_vfull = [&](int st) { return bar + 8 * (1 + 2 * KST + st); };
    auto bar_vempty = [&](int st) { return bar + 8 * (1 + 2 * KST + VST + st); };
    constexpr int B0 = 1 + 2 * KST + 2 * VST;
    auto bar_s = [&](int x) { return bar + 8 * (B0 + x); };        // QK_x done (and all before it)
    auto bar_p = [&](int x) { return bar + 8 * (B0 + 2 + x); };    // P_x written (128 arrivals)
    auto bar_o = [&](int x) { return bar + 8 * (B0 + 4 + x); };    // last PV_x done
    const uint32_t bar_vz = bar + 8 * (B0 + 6);
    const uint32_t bar_fin = bar + 8 * (B0 + 7);
    uint32_t* tm_holder = reinterpret_cast<uint32_t*>(smem + S::OFF_BAR + 256);
    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
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
    auto k_base = [&](int st) { return sm + S::OFF_K + (uint32_t)st * S::KV_BYTES; };
    auto v_base = [&](int st) { return sm + S::OFF_V + (uint32_t)st * S::KV_BYTES; };

    if (warp >= 9) {
        // ===================== TMA producers: warp 9 Q and K, warp 10 V =====================
        const bool is_v = warp == 10;
        int issued = 0;
        if (!is_v && QROWS < S::M) {
            // rows past the tile's queries take zeros (they are never written
            // out; zeros keep their softmax finite and off the redo path)
            const int nz = (S::M - QROWS) * 8;          // 16-byte chunks per 64-dim half
            for (int c = lane; c < (two ? 2 : 1) * S::DH * nz; c += 32) {
                const int x = c / (S::DH * nz), rem = c - x * S::DH * nz;
                const int dh = rem / nz, k = rem - dh * nz;
                *reinterpret_cast<uint4*>(smem + x * S::Q_BYTES + dh * S::Q_HALF + QROWS * 128 + k * 16) =
                    make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async();   // visible to the tensor core's reads of Q
            __syncwarp();
        }
        if (lane == 0 && !is_v) {
            mbar_arrive_expect_tx(bar_q, (uint32_t)((two ? 2 : 1) * S::DH * QROWS * 128));
            for (int x = 0; x < (two ? 2 : 1); ++x)
                for (int dh = 0; dh < S::DH; ++dh)
                    tc05::tma_load_3d(q_base(x) + dh * S::Q_HALF, &tm_q, dh * 64, g * G, q0 + i0 + x * QT, bar_q);
        }
        const int nst = is_v ? VST : KST;
        const CUtensorMap* map = is_v ? &tm_v : &tm_k;
        // Cache row of block bi of tile t, loaded by lane bi (one coalesced load
        // per tile, a tile ahead of its copies); past the sequence's blocks
        // (or for a bad id) the row past the pool, which TMA fills with zeros.
        auto tile_row = [&](int t) -> int {
            int row = p.cache_rows;
            const int lb = t * S::BPT + lane;
            if (lane < S::BPT && lb < nblk_seq) {
                const int phys = __ldg(p.block_tables + (size_t)s * p.max_blocks_per_seq + lb);
                if (phys >= 0 && phys < p.num_blocks) row = (phys * Hkv + g) * BS;
                else if (!is_v) flag_error(p.errors, PKV_DEVERR_BLOCK_ID);
            }
            return row;
        };
        int next_row = tile_row(0);
        for (int t = 0; t < nT; ++t) {
            const int cur_row = next_row;
            if (t + 1 < nT) next_row = tile_row(t + 1);
            const int st = t % nst;
            const uint32_t empty = is_v ? bar_vempty(st) : bar_kempty(st);
            const uint32_t full = is_v ? bar_vfull(st) : bar_kfull(st);
            const uint32_t dst = is_v ? v_base(st) : k_base(st);
            if (t >= nst && !warp_wait(empty, ((t / nst) - 1) & 1, wl)) {
                if (lane == 0) flag_error(p.errors, PKV_DEVERR_WAIT);
                break;
            }
            if (lane == 0) mbar_arrive_expect_tx(full, S::KV_BYTES);
#pragma unroll
            for (int bi = 0; bi < S::BPT; ++bi) {
                const int row = __shfl_sync(kAll, cur_row, bi);
                if (lane == 0)
                    for (int dh = 0; dh < S::DH; ++dh)
                        tc05::tma_load_2d(dst + dh * S::KV_HALF + bi * BS * 128, map, dh * 64, row, full);
            }
            issued = t + 1;
        }
        if (lane == 0) {
            // every copy requested above lands before this warp leaves (the last
            // copy into each stage; earlier ones were consumed before their stage
            // was refilled)
            if (!is_v) mbar_wait_bounded(bar_q, 0, kWaitLimit);
            for (int t = max(0, issued - nst); t < issued; ++t)
                mbar_wait_bounded(is_v ? bar_vfull(t % nst) : bar_kfull(t % nst), (t / nst) & 1, kWaitLimit);
        }
        __syncwarp();
        if (is_v && need_vz && issued == nT) {
            const int st = (nT - 1) % VST;
            if (warp_wait(bar_vfull(st), ((nT - 1) / VST) & 1, wl)) {
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
            bool ok = mbar_wait_bounded(bar_q, 0, wl);
            bool vz_seen = !need_vz;
            auto qk = [&](int x, int i) {                    // S_x = Q_x K_i^T
                const uint32_t d = tm + x * S::TM_TILE + S::TM_S;
                const uint64_t ad = dq + (uint64_t)((x * S::Q_BYTES) >> 4);
                const uint64_t bd = dk + (uint64_t)(((i % KST) * S::KV_BYTES) >> 4);
                // k-th 16-wide slice: +32 bytes inside a swizzle row, next half after 4
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t qoff = ((k >> 2) * S::Q_HALF + (k & 3) * 32) >> 4;
                    const uint32_t koff = ((k >> 2) * S::KV_HALF + (k & 3) * 32) >> 4;
                    tc05::mma_ss(d, ad + qoff, bd + koff, idesc_qk, k > 0 ? 1u : 0u);
                }
                tc05::commit(bar_s(x));
            };
            auto pv = [&](int x, int i) -> bool {            // O_x += P_x V_i
                const int sv = i % VST;
                if (!mbar_wait_bounded(bar_vfull(sv), (i / VST) & 1, wl)) return false;
                if (i == nT - 1 && !vz_seen) {
                    if (!mbar_wait_bounded(bar_vz, 0, wl)) return false;
                    vz_seen = true;
                }
                if (!mbar_wait_bounded(bar_p(x), i & 1, wl)) return false;
                tc05::fence_after_sync();
                const uint32_t base = tm + x * S::TM_TILE;
                const uint64_t vd = dv + (uint64_t)((sv * S::KV_BYTES) >> 4);
                // k-th 16 keys: 16 rows of 128 bytes further; P pairs 8 columns further
#pragma unroll
                for (int k = 0; k < N / 16; ++k)
                    tc05::mma_ts(base + S::TM_O, base + S::TM_S + 8 * k, vd + (uint64_t)(k * 128), idesc_pv,
                                 (i > 0 || k > 0) ? 1u : 0u);
                if (i == nTx(x) - 1) tc05::commit(bar_o(x));
                return true;
            };
            for (int i = 0; ok && i < nT; ++i) {
                if (!mbar_wait_bounded(bar_kfull(i % KST), (i / KST) & 1, wl)) { ok = false; break; }
                tc05::fence_after_sync();
                if (i < nT0) qk(0, i);
                if (two && i >= 1) {                         // V(i-1) last read by PV_1(i-1)
                    if (!pv(1, i - 1)) { ok = false; break; }
                    tc05::commit(bar_vempty((i - 1) % VST));
                }
                if (i < nT1) qk(1, i);
                tc05::commit(bar_kempty(i % KST));
                if (i < nT0) {
                    if (!pv(0, i)) { ok = false; break; }
                    if (!two) tc05::commit(bar_vempty(i % VST));
                }
            }
            if (ok && two) {
                if (pv(1, nT - 1)) tc05::commit(bar_vempty((nT - 1) % VST));
                else ok = false;
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
            const int qi = i0 + x * QT + r / G;         // query of this row
            const bool valid = r < QROWS && qi < n;
            // keys 0 .. pos are visible.  Rows past the sequence's queries are
            // never written and every row's softmax is its own, so they take no
            // mask (a mask there would turn every tile of their warp diagonal)
            const int pos = valid ? L - n + qi : 0x7fffffff;
            const uint32_t trow = tm + x * S::TM_TILE + ((uint32_t)(wq * 32) << 16);
            const float sl2 = p.scale_log2;
            float m_ref = -INFINITY, l = 0.f;           // reference max (log2 units), sum of weights
            for (int i = 0; i < nTme; ++i) {
                if (!warp_wait(bar_s(x), i & 1, wl)) { ok = false; break; }
                tc05::fence_after_sync();
                softmax_tile<T, D>(trow + S::TM_S, trow + S::TM_O, i * N, pos, sl2, i >= 1, m_ref, l);
                tc05::tmem_wait_st();
                tc05::fence_before_sync();
                mbar_arrive(bar_p(x));
            }
            // ---- epilogue: O / l to the output ----
            if (ok && warp_wait(bar_o(x), 0, wl)) {
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
