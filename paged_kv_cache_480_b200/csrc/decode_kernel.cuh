// Paged decode attention for sm_100a: one query token per sequence, keys and
// values in fixed-size physical blocks reached through a block table
// ("Efficient Memory Management for Large Language Model Serving with
// PagedAttention" summary page, section 2: the kernel fetches K/V block by
// block through the block table).
//
// Work decomposition
//   item   = (sequence s, KV head g, partition p): tokens
//            [p * PS, min(L_s, (p + 1) * PS)) of one KV head, for all G query
//            heads of the group (each K/V byte is read from HBM once).
//   warp   = one item at a time.  A warp streams its item's (block, head)
//            K and V tiles -- bs x head_size contiguous bytes each -- into a
//            private ring of R shared-memory stages with untiled bulk copies
//            (TMA engine) completing on one mbarrier per stage; lane 0 issues,
//            all lanes consume.  The next item's table entries and index are
//            fetched one item ahead so the copy stream never stops at item
//            boundaries.
//   grid   = persistent: one CTA per SM, W warps; items beyond the first
//            per warp come from an atomic counter in the workspace (the last
//            warp to finish resets it).
// Arithmetic (all fp32): lane = (token slot u, head h, dim group c); Q lanes
// share a token row, each holding head_size / Q dims of q (pre-scaled by
// scale * log2 e) and of the accumulator.  Dot products reduce over the Q
// lanes with xor shuffles; the online softmax works block-wise in base 2;
// a whole-sequence item writes the normalised output, a partial one writes
// (acc, m, l) for the log-sum-exp merge kernel.
#pragma once

#include "common.cuh"

namespace pkv {

struct DecodeParams {
    void* out;
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    const int32_t* context_lens;
    float* part_acc;        // [items][G][D] unnormalised accumulators
    float2* part_ml;        // [items][G] (m, l), m in log2 units
    int32_t* sched;         // [0] item counter, [1] finished-warp counter
    int32_t* prefix_out;    // [S + 1] partitions before each sequence
    unsigned int* errors;   // sticky device-check bits
    float scale_log2;       // scale * log2(e)
    int num_seqs, num_heads, num_kv_heads, num_blocks, max_blocks_per_seq, max_context_len;
    int partition_size;     // PS tokens, a multiple of block_size, <= 32 blocks
    int stages;             // R
    int warps;              // W consumer warps per CTA
    uint32_t warp_smem;     // bytes of one warp's region
    uint32_t seq_smem;      // bytes of the per-CTA length / prefix arrays
};

template <typename T, int D, int BS, int G>
struct DecodeShape {
    static constexpr int EPC = Elem<T>::kPerChunk;  // elements per 16-byte chunk
    static constexpr int NCH = D / EPC;             // chunks per token row
    static constexpr int Q = (G >= 8) ? 4 : 8;      // lanes per token row
    static constexpr int CPL = NCH / Q;             // chunks per lane
    static constexpr int DL = CPL * EPC;            // dims per lane
    static constexpr int TS = 32 / (Q * G);         // token rows per warp step
    static constexpr int NSTEP = BS / TS;           // warp steps per block
    static constexpr int ROW = D * (int)sizeof(T);  // bytes per token row
    static constexpr int TILE = BS * ROW;           // bytes per (block, KV head) tile
    static constexpr int QBYTES = G * ROW;          // q rows of one group
    static_assert(NCH % Q == 0 && CPL >= 1, "head_size too small for the lane layout");
    static_assert(TS >= 1 && BS % TS == 0, "group size");
};

struct StageMeta {
    int item, s, g, part;
    int nvalid;  // valid tokens in this block (0 = nothing to read)
    int flags;   // kFirst | kLast | kWhole
    int qslot;
    int pad;
};
constexpr int kFirst = 1, kLast = 2, kWhole = 4;

// Host and device agree on this layout of one warp's shared-memory region.
template <typename T, int D, int BS, int G>
struct WarpSmem {
    using S = DecodeShape<T, D, BS, G>;
    __host__ __device__ static constexpr uint32_t ring(int) { return 0; }
    __host__ __device__ static constexpr uint32_t qbuf(int R) { return (uint32_t)R * 2 * S::TILE; }
    __host__ __device__ static constexpr uint32_t meta(int R) {
        return qbuf(R) + (uint32_t)R * S::QBYTES;
    }
    __host__ __device__ static constexpr uint32_t bars(int R) {
        return meta(R) + (uint32_t)R * sizeof(StageMeta);
    }
    __host__ __device__ static constexpr uint32_t bytes(int R) {
        return (bars(R) + (uint32_t)R * 8 + 127) / 128 * 128;
    }
};

struct Item {
    int idx;      // item index (>= n_items: none)
    int s, g, part;
    int tok0;     // first token
    int ntok;     // tokens in the item (may be 0 for an empty sequence)
    int nblk;     // stages the item occupies (>= 1)
    int whole;    // the item is the whole sequence
    int tbl;      // lane j holds the item's j-th physical block id
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <typename T, int D, int BS, int G>
__global__ void __launch_bounds__(256, 1) paged_decode_kernel(const DecodeParams p) {
    using S = DecodeShape<T, D, BS, G>;
    using L = WarpSmem<T, D, BS, G>;
    constexpr unsigned FULL = 0xffffffffu;
    extern __shared__ __align__(128) unsigned char smem[];

    const int nseq = p.num_seqs;
    int* s_len = reinterpret_cast<int*>(smem);   // [S]
    int* s_pre = s_len + nseq;                   // [S + 1]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int R = p.stages;
    unsigned char* wb = smem + p.seq_smem + (size_t)warp * p.warp_smem;
    unsigned char* ring = wb + L::ring(R);
    unsigned char* qbuf = wb + L::qbuf(R);
    StageMeta* meta = reinterpret_cast<StageMeta*>(wb + L::meta(R));
    const uint32_t bar0 = smem_addr(wb + L::bars(R));
    const int PS = p.partition_size;

    // ---- lengths and partition prefix sums (every CTA; CTA 0 publishes) ----
    for (int i = threadIdx.x; i < nseq; i += blockDim.x) {
        int len = p.context_lens[i];
        if (len < 0 || len > p.max_blocks_per_seq * BS || len > p.max_context_len) {
            flag_error(p.errors, PKV_DEVERR_CONTEXT);
            len = 0;
        }
        s_len[i] = len;
    }
    if (lane == 0)
        for (int st = 0; st < R; ++st) mbar_init(bar0 + 8 * st, 1);
    fence_mbar_init();
    __syncthreads();
    if (warp == 0) {
        int carry = 0;
        for (int base = 0; base < nseq; base += 32) {
            const int i = base + lane;
            const int n = (i < nseq) ? max(1, (s_len[i] + PS - 1) / PS) : 0;
            int incl = n;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_up_sync(FULL, incl, off);
                if (lane >= off) incl += v;
            }
            if (i < nseq) s_pre[i] = carry + incl - n;
            carry += __shfl_sync(FULL, incl, 31);
        }
        if (lane == 0) s_pre[nseq] = carry;
    }
    __syncthreads();
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i <= nseq; i += blockDim.x) p.prefix_out[i] = s_pre[i];

    const int Hkv = p.num_kv_heads;
    const int n_items = s_pre[nseq] * Hkv;
    const int NW = gridDim.x * p.warps;
    const int gw = blockIdx.x * p.warps + warp;

    auto fetch = [&](int idx) -> Item {
        Item it;
        it.idx = idx;
        it.s = it.g = it.part = it.tok0 = it.ntok = it.whole = it.tbl = 0;
        it.nblk = 0;
        if (idx >= n_items) return it;
        const int jsp = idx / Hkv;
        it.g = idx - jsp * Hkv;
        int lo = 0, hi = nseq - 1;  // largest s with s_pre[s] <= jsp
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_pre[mid] <= jsp) lo = mid; else hi = mid - 1;
        }
        it.s = lo;
        it.part = jsp - s_pre[lo];
        it.whole = (s_pre[lo + 1] - s_pre[lo]) == 1;
        it.tok0 = it.part * PS;
        it.ntok = min(s_len[lo] - it.tok0, PS);
        const int used = (it.ntok + BS - 1) / BS;
        it.nblk = max(used, 1);
        if (lane < used)
            it.tbl = __ldg(p.block_tables + (size_t)lo * p.max_blocks_per_seq + it.tok0 / BS + lane);
        return it;
    };
    auto next_index = [&]() -> int {
        int v = 0;
        if (lane == 0) v = atomicAdd(p.sched, 1) + NW;
        return __shfl_sync(FULL, v, 0);
    };

    // ---- producer state ----
    Item P = fetch(gw);
    int raw_next = (P.idx < n_items) ? next_index() : n_items;
    Item PN = fetch(raw_next);
    raw_next = (PN.idx < n_items) ? next_index() : n_items;
    int pj = 0;           // next block of P to issue
    int qslot_ctr = 0;    // q slot of P
    int issue_st = 0;
    int issued = 0;
    const size_t tile_elems = (size_t)BS * D;
    const T* kc = reinterpret_cast<const T*>(p.k_cache);
    const T* vc = reinterpret_cast<const T*>(p.v_cache);
    const T* qg = reinterpret_cast<const T*>(p.q);

    auto issue = [&]() {
        if (P.idx >= n_items) return;
        const int st = issue_st;
        const int phys = __shfl_sync(FULL, P.tbl, pj & 31);
        int nvalid = min(max(P.ntok - pj * BS, 0), BS);
        const bool bad = nvalid > 0 && (phys < 0 || phys >= p.num_blocks);
        if (bad) nvalid = 0;
        const bool first = pj == 0, last = pj == P.nblk - 1;
        if (lane == 0) {
            StageMeta m;
            m.item = P.idx; m.s = P.s; m.g = P.g; m.part = P.part;
            m.nvalid = nvalid;
            m.flags = (first ? kFirst : 0) | (last ? kLast : 0) | (P.whole ? kWhole : 0);
            m.qslot = qslot_ctr;
            m.pad = 0;
            meta[st] = m;
            const uint32_t bar = bar0 + 8 * st;
            const uint32_t bytes = (first ? S::QBYTES : 0) + (nvalid > 0 ? 2 * S::TILE : 0);
            mbar_arrive_expect_tx(bar, bytes);
            if (first)
                bulk_g2s(smem_addr(qbuf + qslot_ctr * S::QBYTES),
                         qg + ((size_t)P.s * p.num_heads + (size_t)P.g * G) * D, S::QBYTES, bar);
            if (nvalid > 0) {
                const size_t off = ((size_t)phys * Hkv + P.g) * tile_elems;
                unsigned char* dst = ring + (size_t)st * 2 * S::TILE;
                bulk_g2s(smem_addr(dst), kc + off, S::TILE, bar);
                bulk_g2s(smem_addr(dst + S::TILE), vc + off, S::TILE, bar);
            }
            if (bad) flag_error(p.errors, PKV_DEVERR_BLOCK_ID);
        }
        ++issued;
        issue_st = (st + 1 == R) ? 0 : st + 1;
        if (++pj == P.nblk) {
            P = PN;
            pj = 0;
            qslot_ctr = (qslot_ctr + 1 == R) ? 0 : qslot_ctr + 1;
            PN = fetch(raw_next);
            raw_next = (PN.idx < n_items) ? next_index() : n_items;
        }
    };

    // ---- consumer state ----
    const int c = lane % S::Q;
    const int h = (lane / S::Q) % G;
    const int u = lane / (S::Q * G);
    float qf[S::DL], acc[S::DL];
    float m_run = -INFINITY, l_run = 0.f;
#pragma unroll
    for (int d = 0; d < S::DL; ++d) qf[d] = acc[d] = 0.f;

    for (int i = 0; i < R; ++i) issue();
    int cons_st = 0;
    uint32_t phase = 0;
    int consumed = 0;
    bool lost = false;

    while (consumed < issued) {
        const uint32_t bar = bar0 + 8 * cons_st;
        if (!mbar_wait_bounded(bar, phase, kWaitLimit)) {
            flag_error(p.errors, PKV_DEVERR_WAIT);
            lost = true;
            break;
        }
        const StageMeta mt = meta[cons_st];
        if (mt.flags & kFirst) {
            const uint4* qrow = reinterpret_cast<const uint4*>(qbuf + mt.qslot * S::QBYTES + h * S::ROW);
#pragma unroll
            for (int k = 0; k < S::CPL; ++k) {
                float f[S::EPC];
                Elem<T>::widen(qrow[c + S::Q * k], f);
#pragma unroll
                for (int e = 0; e < S::EPC; ++e) qf[k * S::EPC + e] = f[e] * p.scale_log2;
            }
#pragma unroll
            for (int d = 0; d < S::DL; ++d) acc[d] = 0.f;
            m_run = -INFINITY;
            l_run = 0.f;
        }
        const int nvalid = mt.nvalid;
        if (nvalid > 0) {
            const unsigned char* Kt = ring + (size_t)cons_st * 2 * S::TILE;
            const unsigned char* Vt = Kt + S::TILE;
            float z[S::NSTEP];
#pragma unroll
            for (int i = 0; i < S::NSTEP; ++i) {
                const int t = i * S::TS + u;
                const uint4* row = reinterpret_cast<const uint4*>(Kt + t * S::ROW);
                float s0 = 0.f, s1 = 0.f;
#pragma unroll
                for (int k = 0; k < S::CPL; ++k) {
                    float f[S::EPC];
                    Elem<T>::widen(row[c + S::Q * k], f);
#pragma unroll
                    for (int e = 0; e < S::EPC; e += 2) {
                        s0 = fmaf(qf[k * S::EPC + e], f[e], s0);
                        s1 = fmaf(qf[k * S::EPC + e + 1], f[e + 1], s1);
                    }
                }
                float sc = s0 + s1;
#pragma unroll
                for (int off = 1; off < S::Q; off <<= 1) sc += __shfl_xor_sync(FULL, sc, off);
                z[i] = (t < nvalid) ? sc : -INFINITY;
            }
            float mb = z[0];
#pragma unroll
            for (int i = 1; i < S::NSTEP; ++i) mb = fmaxf(mb, z[i]);
#pragma unroll
            for (int off = S::Q * G; off < 32; off <<= 1) mb = fmaxf(mb, __shfl_xor_sync(FULL, mb, off));
            const float m_new = fmaxf(m_run, mb);   // finite: nvalid > 0
            const float alpha = ex2(m_run - m_new);
            l_run *= alpha;
#pragma unroll
            for (int d = 0; d < S::DL; ++d) acc[d] *= alpha;
#pragma unroll
            for (int i = 0; i < S::NSTEP; ++i) {
                const int t = i * S::TS + u;
                if (t < nvalid) {
                    const float pr = ex2(z[i] - m_new);
                    l_run += pr;
                    const uint4* row = reinterpret_cast<const uint4*>(Vt + t * S::ROW);
#pragma unroll
                    for (int k = 0; k < S::CPL; ++k) {
                        float f[S::EPC];
                        Elem<T>::widen(row[c + S::Q * k], f);
#pragma unroll
                        for (int e = 0; e < S::EPC; ++e)
                            acc[k * S::EPC + e] = fmaf(pr, f[e], acc[k * S::EPC + e]);
                    }
                }
            }
            m_run = m_new;
        }
        if (mt.flags & kLast) {
            float lt = l_run;
#pragma unroll
            for (int off = S::Q * G; off < 32; off <<= 1) {
                lt += __shfl_xor_sync(FULL, lt, off);
#pragma unroll
                for (int d = 0; d < S::DL; ++d) acc[d] += __shfl_xor_sync(FULL, acc[d], off);
            }
            if (u == 0) {
                if (mt.flags & kWhole) {
                    const float inv = lt > 0.f ? 1.f / lt : 0.f;
                    uint4* orow = reinterpret_cast<uint4*>(reinterpret_cast<T*>(p.out) +
                                                           ((size_t)mt.s * p.num_heads + (size_t)mt.g * G + h) * D);
#pragma unroll
                    for (int k = 0; k < S::CPL; ++k) {
                        float f[S::EPC];
#pragma unroll
                        for (int e = 0; e < S::EPC; ++e) f[e] = acc[k * S::EPC + e] * inv;
                        orow[c + S::Q * k] = Elem<T>::narrow(f);
                    }
                } else {
                    float4* prow = reinterpret_cast<float4*>(p.part_acc + ((size_t)mt.item * G + h) * D);
#pragma unroll
                    for (int k = 0; k < S::CPL; ++k)
#pragma unroll
                        for (int e = 0; e < S::EPC; e += 4)
                            prow[((c + S::Q * k) * S::EPC + e) / 4] =
                                make_float4(acc[k * S::EPC + e], acc[k * S::EPC + e + 1],
                                            acc[k * S::EPC + e + 2], acc[k * S::EPC + e + 3]);
                    if (c == 0) p.part_ml[(size_t)mt.item * G + h] = make_float2(m_run, lt);
                }
            }
        }
        __syncwarp();
        ++consumed;
        if (++cons_st == R) { cons_st = 0; phase ^= 1u; }
        issue();
    }

    // Retire: the last warp to finish resets the scheduling counters.
    if (!lost && lane == 0) {
        __threadfence();
        const int done = atomicAdd(p.sched + 1, 1);
        if (done == NW - 1) {
            atomicExch(p.sched, 0);
            atomicExch(p.sched + 1, 0);
        }
    }
}

// ---------------------------------------------------------------------------
// Log-sum-exp merge of the partitions of every sequence that has more than
// one (the exact identity: with M = max_p m_p and w_p = 2^(m_p - M),
// out = sum_p w_p acc_p / sum_p w_p l_p).  One CTA per (sequence, group of
// 4 query heads); each thread owns 4 dims of one head.
// ---------------------------------------------------------------------------
struct ReduceParams {
    void* out;
    const float* part_acc;
    const float2* part_ml;
    const int32_t* prefix;
    int num_seqs, num_heads, num_kv_heads;
};

template <typename T, int D>
__global__ void __launch_bounds__(D) lse_merge_kernel(const ReduceParams p) {
    const int s = blockIdx.x;
    const int np = p.prefix[s + 1] - p.prefix[s];
    if (np <= 1) return;
    const int G = p.num_heads / p.num_kv_heads;
    const int h = blockIdx.y * 4 + threadIdx.x / (D / 4);
    if (h >= p.num_heads) return;
    const int d4 = threadIdx.x % (D / 4);
    const int g = h / G, hh = h % G;
    const int base = p.prefix[s];
    float M = -INFINITY;
    for (int q = 0; q < np; ++q) {
        const size_t item = (size_t)(base + q) * p.num_kv_heads + g;
        M = fmaxf(M, p.part_ml[item * G + hh].x);
    }
    float den = 0.f;
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
        for (int q = 0; q < np; ++q) {
            const size_t item = (size_t)(base + q) * p.num_kv_heads + g;
            const float2 ml = p.part_ml[item * G + hh];
            if (ml.x == -INFINITY) continue;
            const float w = ex2(ml.x - M);
            den = fmaf(w, ml.y, den);
            const float4 a = reinterpret_cast<const float4*>(p.part_acc + (item * G + hh) * D)[d4];
            num.x = fmaf(w, a.x, num.x);
            num.y = fmaf(w, a.y, num.y);
            num.z = fmaf(w, a.z, num.z);
            num.w = fmaf(w, a.w, num.w);
        }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    float f[4] = {num.x * inv, num.y * inv, num.z * inv, num.w * inv};
    T* o = reinterpret_cast<T*>(p.out) + ((size_t)s * p.num_heads + h) * D + d4 * 4;
#pragma unroll
    for (int e = 0; e < 4; ++e) o[e] = static_cast<T>(f[e]);
}

}  // namespace pkv
