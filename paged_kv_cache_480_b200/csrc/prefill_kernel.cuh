// Paged prefill / chunked-prefill attention on the sm_100a tensor cores
// (tcgen05 MMA, accumulators in tensor memory, operands staged by TMA).
//
// Sequence s holds L = context_lens[s] tokens in its blocks; the last n of
// them are this call's queries (rows query_start_loc[s] .. +n of q), query i
// at position L - n + i attending causally to keys 0 .. L - n + i ("PyTorch-
// CUDA-v2.9 image enables PagedAttention", workflow list: prefill writes the
// prompt's KV into pages; usage: chunked prefill).
//
// Work item = (sequence, KV head g, two query tiles of M = 128 rows each); a
// row is a (query, head-of-group) pair, row = query * G + head, so every K/V
// tile serves the G query heads that share it, and both query tiles of the
// item share each K/V tile brought into shared memory.  A query tile holds
// QT = floor(128 / G) queries; when G does not divide 128 its last
// 128 - QT * G rows are zero and never written out.
//
// The grid is persistent: one CTA per SM takes items from a counter, in
// groups of (sequence, KV head) pairs whose K/V fits in half of L2, the
// tiles with most keys first inside a group.  A CTA's K/V streams and its
// tensor-core pipeline run on from one item into the next: the next item's
// q tile x is loaded as soon as the current item's last product with q tile
// x is done, and query tile x's output is written out while the other tile
// works.  Roles:
//   warps 0-3 and 4-7  softmax and output of query tile 0 and 1, one row per
//                      thread (warp w reaches tensor-memory lanes 32(w%4) .. +31);
//   warp 8             issues the MMAs (one thread);
//   warps 9 and 10     stream K and V tiles through two rings of stages with
//                      TMA, each refilling a stage once the products that
//                      read it are done; warp 10 also zeroes the V rows past
//                      a context's end in its last block;
//   warp 11            takes items from the counter, hands them to the other
//                      roles through a ring in shared memory, and loads q.
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
// units, so O stays exact up to the final division by l (tc_softmax.cuh).
// Masks are applied only on tiles that reach past some row's position.
// Every wait is bounded; the tensor memory is freed on every path.
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
    int* sched;                       // [0] item counter, [1] finished CTAs (zero between launches)
    float scale_log2;                 // softmax scale * log2(e), > 0
    int num_tokens, num_seqs, num_heads, num_kv_heads, num_blocks, max_blocks_per_seq;
    int group;                        // G = num_heads / num_kv_heads, 1 .. 128
    int qt;                           // queries per query tile: floor(128 / G)
    uint32_t wait_limit;              // polls before a wait for progress gives up
    int q_tiles;                      // items (query-tile pairs) per (sequence, KV head)
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
    static constexpr int IR = 2;                // items in flight between the roles (one ahead: a deeper
                                                // ring lets CTAs claim items further ahead, spreading
                                                // the L2 groups: chunked reads +5%)
    static constexpr uint32_t Q_HALF = M * 128;
    static constexpr uint32_t KV_HALF = N * 128;
    static constexpr uint32_t Q_BYTES = DH * Q_HALF;        // one query tile
    static constexpr uint32_t KV_BYTES = DH * KV_HALF;      // K or V of one key tile
    static constexpr uint32_t OFF_K = 2 * Q_BYTES;
    static constexpr uint32_t OFF_V = OFF_K + KST * KV_BYTES;
    static constexpr uint32_t OFF_BAR = OFF_V + VST * KV_BYTES;
    static constexpr uint32_t NBAR = 2 * IR + 4 + 2 * (KST + VST) + 10;
    static constexpr uint32_t OFF_ITEMS = (OFF_BAR + 8 * NBAR + 63) / 64 * 64;   // item ring, 64 bytes a slot
    static constexpr uint32_t OFF_HOLD = OFF_ITEMS + 64 * IR;                   // tensor-memory address
    static constexpr uint32_t SMEM = OFF_HOLD + 16 + 1024;  // 1 KB alignment slack
    static constexpr uint32_t TM_TILE = 256;                // columns per query tile
    static constexpr uint32_t TM_S = 0;                     // S (N fp32 columns); P over its first N/2
    static constexpr uint32_t TM_O = N;                     // O at columns N .. N + D
    static constexpr uint32_t TM_COLS = 512;
    static_assert(N + D <= (int)TM_TILE, "tensor-memory budget");
    static_assert(N % BS == 0, "key tile holds whole blocks");
    static_assert(SMEM > 232448 / 2 && SMEM <= 232448, "one CTA per SM");
};

constexpr uint32_t kPrefillThreads = 384;

// One work item as the scheduler hands it to the other roles.
struct PrefillItem {
    int s, g;              // sequence, KV head (s < 0: no more items)
    int q0, n, L;          // first q row of the sequence, its queries, its tokens
    int i0;                // first query of the item (query tile 0; tile 1 starts QT later)
    int nT0, nT1;          // key tiles of query tile 0 and 1 (0: no query)
    int vz_r0, vz_r1;      // V rows of the item's last key tile to zero (r0 >= r1: none)
    int pad[6];
};
static_assert(sizeof(PrefillItem) == 64, "item slot");

template <typename T, int D, int BS>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    paged_prefill_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
    using S = PrefillShape<T, D, BS>;
    using namespace tcsm;
    constexpr int KST = S::KST, VST = S::VST, IR = S::IR;
    constexpr int N = S::N;
    constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw_s = smem_addr(smem_raw);
    const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
    unsigned char* smem = smem_raw + pad;
    const uint32_t sm = raw_s + pad;                // 1024-byte aligned shared address
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.group, QT = p.qt, CQ = 2 * QT;  // heads per KV head; queries per tile and per item
    const int QROWS = QT * G;                       // rows of a query tile that hold queries
    const uint32_t wl = p.wait_limit;
    const int Hkv = p.num_kv_heads;

    // ---- barriers, item ring, tensor memory ----
    const uint32_t bar = sm + S::OFF_BAR;
    auto bar_ifull = [&](int k) { return bar + 8 * k; };               // item slot written
    auto bar_iempty = [&](int k) { return bar + 8 * (IR + k); };       // item slot read by every role
    auto bar_qfull = [&](int x) { return bar + 8 * (2 * IR + x); };
    auto bar_qempty = [&](int x) { return bar + 8 * (2 * IR + 2 + x); };   // an item's last QK_x done
    constexpr int BK = 2 * IR + 4;
    auto bar_kfull = [&](int st) { return bar + 8 * (BK + st); };
    auto bar_kempty = [&](int st) { return bar + 8 * (BK + KST + st); };
    auto bar_vfull = [&](int st) { return bar + 8 * (BK + 2 * KST + st); };
    auto bar_vempty = [&](int st) { return bar + 8 * (BK + 2 * KST + VST + st); };
    constexpr int B0 = BK + 2 * KST + 2 * VST;
    auto bar_s = [&](int x) { return bar + 8 * (B0 + x); };          // QK_x done (and all before it)
    auto bar_p = [&](int x) { return bar + 8 * (B0 + 2 + x); };      // P_x written (128 arrivals)
    auto bar_o = [&](int x) { return bar + 8 * (B0 + 4 + x); };      // an item's last PV_x done
    auto bar_ofree = [&](int x) { return bar + 8 * (B0 + 6 + x); };  // O_x written out (128 arrivals)
    const uint32_t bar_vz = bar + 8 * (B0 + 8);
    const uint32_t bar_fin = bar + 8 * (B0 + 9);
    PrefillItem* items = reinterpret_cast<PrefillItem*>(smem + S::OFF_ITEMS);
    uint32_t* tm_holder = reinterpret_cast<uint32_t*>(smem + S::OFF_HOLD);
    constexpr int kItemReaders = 11;                // warps 0-7, and warps 8, 9, 10 once each
    if (threadIdx.x == 0) {
        for (int k = 0; k < IR; ++k) {
            mbar_init(bar_ifull(k), 1);
            mbar_init(bar_iempty(k), kItemReaders);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(bar_qfull(x), 1);
            mbar_init(bar_qempty(x), 1);
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
    if (QROWS < S::M) {
        // rows past a tile's queries stay zero in both q buffers (the q box never
        // writes them; zeros keep their softmax finite and off the redo path)
        const int nz = (S::M - QROWS) * 8;          // 16-byte chunks per 64-dim half
        for (int i = threadIdx.x; i < 2 * S::DH * nz; i += blockDim.x) {
            const int h = i / nz, k = i - h * nz;   // h = query tile * DH + dh
            *reinterpret_cast<uint4*>(smem + h * S::Q_HALF + QROWS * 128 + k * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async();   // visible to the tensor core's reads of Q
    }
    tc05::fence_before_sync();
    __syncthreads();
    tc05::fence_after_sync();
    const uint32_t tm = *tm_holder;
    griddep_wait();

    auto q_base = [&](int x) { return sm + (uint32_t)x * S::Q_BYTES; };
    auto k_base = [&](int st) { return sm + S::OFF_K + (uint32_t)st * S::KV_BYTES; };
    auto v_base = [&](int st) { return sm + S::OFF_V + (uint32_t)st * S::KV_BYTES; };
    // Item j of this CTA from the ring, taken by a whole warp (its lane 0 arrives
    // on the slot's empty barrier).
    auto take_item = [&](int j, PrefillItem& it) -> bool {
        if (!warp_wait(bar_ifull(j % IR), (j / IR) & 1, wl)) return false;
        it = items[j % IR];
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_iempty(j % IR));
        return true;
    };

    if (warp == 11) {
        // ===================== scheduler: items from the counter, q by TMA =====================
        const int pairs = p.num_seqs * Hkv;
        const int gp = min(p.sched_group, pairs);
        const int per_group = gp * p.q_tiles;
        const int n_items = pairs * p.q_tiles;
        int idx = blockIdx.x, j = 0, qloads[2] = {0, 0};
        bool ok = true;
        auto next_index = [&]() {
            int v = 0;
            if (lane == 0) v = atomicAdd(p.sched, 1) + (int)gridDim.x;
            idx = __shfl_sync(kAll, v, 0);
        };
        while (true) {
            PrefillItem it;
            it.s = -1;
            if (idx < n_items) {
                // groups of p.sched_group (sequence, KV head) pairs, one after the
                // other; inside a group the tiles with most keys go first.  The
                // host sizes groups so that a group's K/V fits in half of L2 while
                // its query tiles read it.
                const int grp = idx / per_group;
                const int in_g = idx - grp * per_group;
                const int g_pairs = min(gp, pairs - grp * gp);   // the last group may be smaller
                const int tile = p.q_tiles - 1 - in_g / g_pairs;
                const int rest = grp * gp + in_g % g_pairs;
                const int s = rest / Hkv;
                const int q0 = __ldg(p.query_start_loc + s);
                const int n = __ldg(p.query_start_loc + s + 1) - q0;
                const int L = __ldg(p.context_lens + s);
                const int i0 = tile * CQ;
                if (n < 0 || n > L || n > p.q_tiles * CQ || L > p.max_blocks_per_seq * BS || q0 < 0 ||
                    q0 + n > p.num_tokens) {
                    // a bad sequence is skipped (its rows are not written) and flagged
                    if (lane == 0 && tile == p.q_tiles - 1) flag_error(p.errors, PKV_DEVERR_CONTEXT);
                    next_index();
                    continue;
                }
                if (i0 >= n) {                  // a query-tile pair past the sequence's queries
                    next_index();
                    continue;
                }
                it.s = s;
                it.g = rest - s * Hkv;
                it.q0 = q0;
                it.n = n;
                it.L = L;
                it.i0 = i0;
                // key tiles each query tile needs (0: the tile holds no query)
                it.nT0 = (L - n + min(i0 + QT, n) + N - 1) / N;
                it.nT1 = i0 + QT < n ? (L - n + min(i0 + CQ, n) + N - 1) / N : 0;
                const int nT = max(it.nT0, it.nT1);
                const int nblk = (L + BS - 1) / BS;
                it.vz_r0 = L - (nT - 1) * N;
                it.vz_r1 = min(nblk * BS - (nT - 1) * N, N);
            }
            // hand the item (or the end mark) to the other roles
            const int k = j % IR;
            if (j >= IR && !warp_wait(bar_iempty(k), ((j / IR) - 1) & 1, wl)) { ok = false; break; }
            if (lane == 0) {
                items[k] = it;
                mbar_arrive(bar_ifull(k));          // release: the slot's contents before the arrival
            }
            __syncwarp();
            ++j;
            if (it.s < 0) break;
            // q of the item's tiles, once the previous item's products with them are done
            for (int x = 0; x < (it.nT1 > 0 ? 2 : 1); ++x) {
                if (qloads[x] >= 1 && !warp_wait(bar_qempty(x), (qloads[x] - 1) & 1, wl)) { ok = false; break; }
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar_qfull(x), (uint32_t)(S::DH * QROWS * 128));
                    for (int dh = 0; dh < S::DH; ++dh)
                        tc05::tma_load_3d(q_base(x) + dh * S::Q_HALF, &tm_q, dh * 64, it.g * G,
                                          it.q0 + it.i0 + x * QT, bar_qfull(x));
                }
                ++qloads[x];
            }
            if (!ok) break;
            next_index();
        }
        // (if a wait gave up here, the other roles' own bounded waits give up too)
        if (!ok && lane == 0) flag_error(p.errors, PKV_DEVERR_WAIT);
        // every q copy requested above lands before this warp leaves
        if (lane == 0)
            for (int x = 0; x < 2; ++x)
                if (qloads[x] > 0) mbar_wait_bounded(bar_qfull(x), (qloads[x] - 1) & 1, kWaitLimit);
        __syncwarp();
    } else if (warp >= 9) {
        // ===================== TMA producers: warp 9 K, warp 10 V =====================
        const bool is_v = warp == 10;
        const int nst = is_v ? VST : KST;
        const CUtensorMap* map = is_v ? &tm_v : &tm_k;
        int jt = 0;                                  // key tiles streamed so far
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
        for (int j = 0; ok; ++j) {
            PrefillItem it;
            if (!take_item(j, it)) { ok = false; break; }
            if (it.s < 0) break;
            const int s = it.s, g = it.g;
            const int nT = max(it.nT0, it.nT1);
            const int nblk = (it.L + BS - 1) / BS;
            // cache row of block `lane` of key tile t (one coalesced load per tile,
            // a tile ahead of its copies); past the sequence's blocks, or for a
            // bad id, the row past the pool, which TMA fills with zeros
            auto tile_row = [&](int t) -> int {
                int row = p.cache_rows;
                const int lb = t * S::BPT + lane;
                if (lane < S::BPT && lb < nblk) {
                    const int phys = __ldg(p.block_tables + (size_t)s * p.max_blocks_per_seq + lb);
                    if (phys >= 0 && phys < p.num_blocks) row = (phys * Hkv + g) * BS;
                    else if (!is_v) flag_error(p.errors, PKV_DEVERR_BLOCK_ID);
                }
                return row;
            };
            int next_row = tile_row(0);
            for (int t = 0; t < nT; ++t, ++jt) {
                const int cur_row = next_row;
                if (t + 1 < nT) next_row = tile_row(t + 1);
                const int st = jt % nst;
                // a pending zeroing happens before its stage is waited for again
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
                // the item's last key tile: V rows from the context end to the end
                // of its last block hold whatever the pool holds there
                if (is_v && t == nT - 1 && it.vz_r0 < it.vz_r1) {
                    if (vz_jt >= 0) do_vz();
                    vz_jt = jt;
                    vz_r0 = it.vz_r0;
                    vz_r1 = it.vz_r1;
                }
            }
        }
        if (is_v && vz_jt >= 0 && ok) do_vz();
        if (!ok && lane == 0) flag_error(p.errors, PKV_DEVERR_WAIT);
        if (lane == 0) {
            // every copy requested above lands before this warp leaves (the last
            // copy into each stage; earlier ones were consumed before their stage
            // was refilled)
            for (int t = max(0, jt - nst); t < jt; ++t)
                mbar_wait_bounded(is_v ? bar_vfull(t % nst) : bar_kfull(t % nst), (t / nst) & 1, kWaitLimit);
        }
        __syncwarp();
    } else if (warp == 8) {
        // ===================== MMA issue (one thread) =====================
        if (lane == 0) {
            constexpr uint32_t idesc_qk = tc05::instr_desc(kBf16, 128, N, false, false);
            constexpr uint32_t idesc_pv = tc05::instr_desc(kBf16, 128, D, false, true);
            // operand descriptors of query tile 0 and stage 0; the start-address
            // field (bits 0-13, address / 16) is advanced by plain addition
            const uint64_t dq = tc05::smem_desc(q_base(0), 16, 1024);
            const uint64_t dk = tc05::smem_desc(k_base(0), 16, 1024);
            const uint64_t dv = tc05::smem_desc(v_base(0), S::KV_HALF, 1024);
            bool ok = true;
            int jt0 = 0, vzc = 0;                          // key tiles of earlier items; zeroings seen
            int qx[2] = {0, 0}, px[2] = {0, 0}, ox[2] = {0, 0};   // q loads, P phases, items per tile
            for (int j = 0; ok; ++j) {
                if (!mbar_wait_bounded(bar_ifull(j % IR), (j / IR) & 1, wl)) { ok = false; break; }
                const PrefillItem it = items[j % IR];
                mbar_arrive(bar_iempty(j % IR));
                if (it.s < 0) break;
                const int nT0 = it.nT0, nT1 = it.nT1, nT = max(nT0, nT1);
                const bool two = nT1 > 0;
                const bool vz = it.vz_r0 < it.vz_r1;
                const int vz_x = nT0 == nT ? 0 : 1;            // the first product reading the last V tile
                auto qk = [&](int x, int i) {                  // S_x = Q_x K_i^T
                    const uint32_t d = tm + x * S::TM_TILE + S::TM_S;
                    const uint64_t ad = dq + (uint64_t)((x * S::Q_BYTES) >> 4);
                    const uint64_t bd = dk + (uint64_t)((((jt0 + i) % KST) * S::KV_BYTES) >> 4);
                    // k-th 16-wide slice: +32 bytes inside a swizzle row, next half after 4
#pragma unroll
                    for (int k = 0; k < D / 16; ++k) {
                        const uint32_t qoff = ((k >> 2) * S::Q_HALF + (k & 3) * 32) >> 4;
                        const uint32_t koff = ((k >> 2) * S::KV_HALF + (k & 3) * 32) >> 4;
                        tc05::mma_ss(d, ad + qoff, bd + koff, idesc_qk, k > 0 ? 1u : 0u);
                    }
                    tc05::commit(bar_s(x));
                    if (i == (x ? nT1 : nT0) - 1) tc05::commit(bar_qempty(x));   // Q_x free for the next item
                };
                auto pv = [&](int x, int i) -> bool {          // O_x += P_x V_i
                    const int jt = jt0 + i, sv = jt % VST;
                    if (!mbar_wait_bounded(bar_vfull(sv), (jt / VST) & 1, wl)) return false;
                    if (vz && i == nT - 1 && x == vz_x) {
                        if (!mbar_wait_bounded(bar_vz, vzc & 1, wl)) return false;
                        ++vzc;
                    }
                    if (!mbar_wait_bounded(bar_p(x), px[x] & 1, wl)) return false;
                    ++px[x];
                    if (i == 0) {
                        // the tile's previous item must be written out before O_x restarts
                        if (ox[x] >= 1 && !mbar_wait_bounded(bar_ofree(x), (ox[x] - 1) & 1, wl)) return false;
                        ++ox[x];
                    }
                    tc05::fence_after_sync();
                    const uint32_t base = tm + x * S::TM_TILE;
                    const uint64_t vd = dv + (uint64_t)((sv * S::KV_BYTES) >> 4);
                    // k-th 16 keys: 16 rows of 128 bytes further; P pairs 8 columns further
#pragma unroll
                    for (int k = 0; k < N / 16; ++k)
                        tc05::mma_ts(base + S::TM_O, base + S::TM_S + 8 * k, vd + (uint64_t)(k * 128), idesc_pv,
                                     (i > 0 || k > 0) ? 1u : 0u);
                    if (i == (x ? nT1 : nT0) - 1) tc05::commit(bar_o(x));
                    return true;
                };
                if (!mbar_wait_bounded(bar_qfull(0), qx[0] & 1, wl)) { ok = false; break; }
                ++qx[0];
                for (int i = 0; ok && i < nT; ++i) {
                    const int jt = jt0 + i;
                    if (!mbar_wait_bounded(bar_kfull(jt % KST), (jt / KST) & 1, wl)) { ok = false; break; }
                    tc05::fence_after_sync();
                    if (i < nT0) qk(0, i);
                    if (two && i >= 1) {                       // V(i-1) last read by PV_1(i-1)
                        if (!pv(1, i - 1)) { ok = false; break; }
                        tc05::commit(bar_vempty((jt - 1) % VST));
                    }
                    if (i < nT1) {
                        if (i == 0) {                           // q tile 1 is needed from here on
                            if (!mbar_wait_bounded(bar_qfull(1), qx[1] & 1, wl)) { ok = false; break; }
                            ++qx[1];
                        }
                        qk(1, i);
                    }
                    tc05::commit(bar_kempty(jt % KST));
                    if (i < nT0) {
                        if (!pv(0, i)) { ok = false; break; }
                        if (!two) tc05::commit(bar_vempty(jt % VST));
                    }
                }
                if (ok && two) {
                    if (pv(1, nT - 1)) tc05::commit(bar_vempty((jt0 + nT - 1) % VST));
                    else ok = false;
                }
                jt0 += nT;
            }
            if (!ok) flag_error(p.errors, PKV_DEVERR_WAIT);
            // every MMA issued above is complete before the tensor memory is freed
            tc05::commit(bar_fin);
            mbar_wait_bounded(bar_fin, 0, kWaitLimit);
        }
    } else {
        // ===================== softmax and output: one row per thread =====================
        const int x = warp >> 2;                        // query tile
        const int wq = warp & 3;
        const int r = wq * 32 + lane;                   // row within the tile
        const uint32_t trow = tm + x * S::TM_TILE + ((uint32_t)(wq * 32) << 16);
        const float sl2 = p.scale_log2;
        int nx = 0, ox = 0;                             // S_x phases; items with this tile
        bool ok = true;
        for (int j = 0; ok; ++j) {
            PrefillItem it;
            if (!take_item(j, it)) { ok = false; break; }
            if (it.s < 0) break;
            const int nTme = x ? it.nT1 : it.nT0;
            if (nTme == 0) continue;
            const int n = it.n, L = it.L;
            const int qi = it.i0 + x * QT + r / G;      // query of this row
            const bool valid = r < QROWS && qi < n;
            // keys 0 .. pos are visible.  Rows past the sequence's queries are
            // never written and every row's softmax is its own, so they take no
            // mask (a mask there would turn every tile of their warp diagonal)
            const int pos = valid ? L - n + qi : 0x7fffffff;
            float m_ref = -INFINITY, l = 0.f;           // reference max (log2 units), sum of weights
            for (int i = 0; i < nTme; ++i) {
                if (!warp_wait(bar_s(x), nx & 1, wl)) { ok = false; break; }
                ++nx;
                tc05::fence_after_sync();
                softmax_tile<T, D>(trow + S::TM_S, trow + S::TM_O, i * N, pos, sl2, i >= 1, m_ref, l);
                tc05::tmem_wait_st();
                tc05::fence_before_sync();
                mbar_arrive(bar_p(x));
            }
            // ---- O / l to the output ----
            if (ok && warp_wait(bar_o(x), ox & 1, wl)) {
                tc05::fence_after_sync();
                const float inv = l > 0.f ? 1.f / l : 0.f;
                T* orow = reinterpret_cast<T*>(p.out) +
                          ((size_t)(it.q0 + qi) * p.num_heads + (size_t)it.g * G + (r % G)) * D;
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
                tc05::fence_before_sync();
                mbar_arrive(bar_ofree(x));
            } else {
                ok = false;
            }
            ++ox;
        }
        if (!ok && lane == 0) flag_error(p.errors, PKV_DEVERR_WAIT);
    }
    griddep_launch();
    tc05::fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc05::fence_after_sync();
        tc05::tmem_dealloc(tm, S::TM_COLS);
    }
    // the last CTA to finish resets the item counter for the next launch that uses it
    if (threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(p.sched + 1, 1) == (int)gridDim.x - 1) {
            atomicExch(p.sched, 0);
            atomicExch(p.sched + 1, 0);
        }
    }
}

}  // namespace pkv
