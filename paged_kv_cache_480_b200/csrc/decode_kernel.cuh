// Paged decode attention for sm_100a: one query token per sequence, keys and
// values in fixed-size physical blocks reached through a block table
// ("Efficient Memory Management for Large Language Model Serving with
// PagedAttention" summary page, section 2: the kernel fetches K/V block by
// block through the block table).
//
// Work decomposition
//   item   = (sequence s, KV head g, partition p, head slice): tokens
//            [p * PS, min(L_s, (p + 1) * PS)) of one KV head, for the query
//            heads of the group (each K/V byte is read from HBM once).  A
//            group of up to 8 query heads is one slice, padded to the kernel's
//            column count GP in {1, 2, 4, 8}; a larger group is split into
//            slices of 8 heads whose items follow each other, so their warps
//            stream the same tiles at about the same time and all but the
//            first read them from L2.
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
//
// The arithmetic of a stage is a consumer type:
//   FmaConsumer  fp32 CUDA-core FMAs (every element type, small groups);
//   MmaConsumer  tensor-core mma.m16n8k16 for groups of 4-8 query heads with
//                16-bit elements, where the fp32 FMA issue rate, not HBM,
//                would bound the kernel.
// Both keep a base-2 online softmax per head; a whole-sequence item writes
// the normalised output, a partial one writes (acc, m, l) for the
// log-sum-exp merge kernel (merge_kernel.cuh).
#pragma once

#include <type_traits>

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
    float k_scale, v_scale; // cache element = real value / scale (1 unless the cache is FP8)
    int num_seqs, num_heads, num_kv_heads, num_blocks, max_blocks_per_seq, max_context_len;
    int partition_size;     // PS tokens, a multiple of block_size, <= 32 blocks
    int partition_min;      // > 0: choose PS in [partition_min, partition_size] on the device
    // Fused cache write (all null for a plain decode): the step's new token
    // of sequence s, rows key[s][g] / value[s][g], goes to slot
    // slot_mapping[s], which must be the slot of position context_len - 1.
    const void* key;
    const void* value;
    const int64_t* slot_mapping;
    int64_t key_stride, value_stride;   // elements between sequences
    int group;              // G = num_heads / num_kv_heads (any value >= 1)
    int slices;             // head slices per group: ceil(G / GP)
    uint32_t wait_limit;    // polls before a wait for a stage's copies gives up
    int stages;             // R
    int warps;              // W consumer warps per CTA
    uint32_t warp_smem;     // bytes of one warp's region
    uint32_t seq_smem;      // bytes of the per-CTA length / prefix arrays
};

// TQ: element type of q and out; TC: element type of the caches; G: query-head
// columns of one item (the group size padded to 1, 2, 4 or 8).
template <typename TQ, typename TC, int D, int BS, int G>
struct DecodeShape {
    static constexpr int EPC = Elem<TC>::kPerChunk;  // cache elements per 16-byte chunk
    static constexpr int ROW = D * (int)sizeof(TC);  // bytes per cache token row
    static constexpr int TILE = BS * ROW;            // bytes per (block, KV head) tile
    static constexpr int QROW = D * (int)sizeof(TQ); // bytes per q / out row
    static constexpr int QBYTES = G * QROW;          // q rows of one item, at most
};

struct StageMeta {
    int64_t pidx;   // first partial row of the item: partition index * num_heads + first head
    int64_t obase;  // first output row: s * num_heads + first head
    int64_t slot;   // fused cache write: the new token's slot
    int g;          // KV head
    int nh;         // query heads of the item (<= GP)
    int nvalid;     // valid tokens in this block (0 = nothing to read)
    int flags;      // kFirst | kLast | kWhole | kStore
    int qslot;
    int newrow;     // row of this block that takes the step's new token, or -1
};
// kStore: this item also stores the step's new token into the cache (one
// head slice of a group does)
constexpr int kFirst = 1, kLast = 2, kWhole = 4, kStore = 8;

// Host and device agree on this layout of one warp's shared-memory region.
template <typename TQ, typename TC, int D, int BS, int G>
struct WarpSmem {
    using S = DecodeShape<TQ, TC, D, BS, G>;
    __host__ __device__ static constexpr uint32_t ring(int) { return 0; }
    __host__ __device__ static constexpr uint32_t qbuf(int R) { return (uint32_t)R * 2 * S::TILE; }
    // new-token K and V rows of each stage (fused cache write)
    __host__ __device__ static constexpr uint32_t nbuf(int R) {
        return qbuf(R) + (uint32_t)R * S::QBYTES;
    }
    __host__ __device__ static constexpr uint32_t meta(int R) {
        return nbuf(R) + (uint32_t)R * 2 * S::ROW;
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
    int s;
    int vg;       // KV head * slices + head slice
    int jsp;      // partition index over the batch (partitions of sequences before s, plus this one's)
    int tok0;     // first token
    int ntok;     // tokens in the item (may be 0 for an empty sequence)
    int nblk;     // stages the item occupies (>= 1)
    int whole;    // the item is the whole sequence
    int tbl;      // lane j holds the item's (32k + j)-th physical block id (k = issued blocks / 32)
    int64_t slot; // fused cache write: slot of the new token if this item holds it, else -1
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

constexpr unsigned kFull = 0xffffffffu;

// ===========================================================================
// fp32 CUDA-core consumer.
// lane = (token slot u, head h, dim group c); Q lanes share a token row, each
// holding D / Q dims of q (pre-scaled by scale * log2 e) and of the
// accumulator; dot products reduce over the Q lanes with xor shuffles.  The 8
// lanes of a quarter-warp read one 128-byte segment of a row (no bank
// conflicts).
// ===========================================================================
template <typename TQ, typename TC, int D, int BS, int G>
struct FmaConsumer {
    static constexpr bool kPairs = false;   // one block per consumer step
    using S = DecodeShape<TQ, TC, D, BS, G>;
    static constexpr int EPC = S::EPC;
    static constexpr int EPQ = Elem<TQ>::kPerChunk;  // q / out elements per 16-byte chunk
    static constexpr int QPC = EPC / EPQ;           // q chunks per cache chunk
    static constexpr int NCH = D / EPC;             // chunks per token row
    static constexpr int Q0 = (G >= 8) ? 4 : 8;
    static constexpr int Q = Q0 < NCH ? Q0 : NCH;   // lanes per token row
    static constexpr int CPL = NCH / Q;             // chunks per lane
    static constexpr int DL = CPL * EPC;            // dims per lane
    static constexpr int TS = 32 / (Q * G);         // token rows per warp step
    static constexpr int NSTEP = BS / TS;           // warp steps per block
    static_assert(NCH % Q == 0 && CPL >= 1, "head_size too small for the lane layout");
    static_assert(TS >= 1 && BS % TS == 0, "group size");

    int c, h, u;
    float qf[DL], acc[DL];
    float m_run, l_run;

    __device__ __forceinline__ void init(int lane) {
        c = lane % Q;
        h = (lane / Q) % G;
        u = lane / (Q * G);
        m_run = -INFINITY;
        l_run = 0.f;
#pragma unroll
        for (int d = 0; d < DL; ++d) qf[d] = acc[d] = 0.f;
    }

    // nh: heads of the item; lanes of the padding heads hold q = 0 and write nothing
    __device__ __forceinline__ void begin(const unsigned char* qslot, float qscale, int nh) {
        const uint4* qrow = reinterpret_cast<const uint4*>(qslot + h * S::QROW);
#pragma unroll
        for (int k = 0; k < CPL; ++k)
#pragma unroll
            for (int j = 0; j < QPC; ++j) {
                float f[EPQ];
                if (h < nh) {
                    Elem<TQ>::widen(qrow[(c + Q * k) * QPC + j], f);
                } else {
#pragma unroll
                    for (int e = 0; e < EPQ; ++e) f[e] = 0.f;
                }
#pragma unroll
                for (int e = 0; e < EPQ; ++e) qf[k * EPC + j * EPQ + e] = f[e] * qscale;
            }
#pragma unroll
        for (int d = 0; d < DL; ++d) acc[d] = 0.f;
        m_run = -INFINITY;
        l_run = 0.f;
    }

    __device__ __forceinline__ void block(const unsigned char* Kt, const unsigned char* Vt,
                                          int nvalid, float) {
        float z[NSTEP];
#pragma unroll
        for (int i = 0; i < NSTEP; ++i) {
            const int t = i * TS + u;
            const uint4* row = reinterpret_cast<const uint4*>(Kt + t * S::ROW);
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int k = 0; k < CPL; ++k) {
                float f[EPC];
                Elem<TC>::widen(row[c + Q * k], f);
#pragma unroll
                for (int e = 0; e < EPC; e += 2) {
                    s0 = fmaf(qf[k * EPC + e], f[e], s0);
                    s1 = fmaf(qf[k * EPC + e + 1], f[e + 1], s1);
                }
            }
            float sc = s0 + s1;
#pragma unroll
            for (int off = 1; off < Q; off <<= 1) sc += __shfl_xor_sync(kFull, sc, off);
            z[i] = (t < nvalid) ? sc : -INFINITY;
        }
        float mb = z[0];
#pragma unroll
        for (int i = 1; i < NSTEP; ++i) mb = fmaxf(mb, z[i]);
#pragma unroll
        for (int off = Q * G; off < 32; off <<= 1) mb = fmaxf(mb, __shfl_xor_sync(kFull, mb, off));
        const float m_new = fmaxf(m_run, mb);   // finite: nvalid > 0
        const float alpha = ex2(m_run - m_new);
        l_run *= alpha;
#pragma unroll
        for (int d = 0; d < DL; ++d) acc[d] *= alpha;
#pragma unroll
        for (int i = 0; i < NSTEP; ++i) {
            const int t = i * TS + u;
            if (t < nvalid) {
                const float pr = ex2(z[i] - m_new);
                l_run += pr;
                const uint4* row = reinterpret_cast<const uint4*>(Vt + t * S::ROW);
#pragma unroll
                for (int k = 0; k < CPL; ++k) {
                    float f[EPC];
                    Elem<TC>::widen(row[c + Q * k], f);
#pragma unroll
                    for (int e = 0; e < EPC; ++e) acc[k * EPC + e] = fmaf(pr, f[e], acc[k * EPC + e]);
                }
            }
        }
        m_run = m_new;
    }

    __device__ __forceinline__ void finish(const StageMeta& mt, const DecodeParams& p) {
        float lt = l_run;
#pragma unroll
        for (int off = Q * G; off < 32; off <<= 1) {
            lt += __shfl_xor_sync(kFull, lt, off);
#pragma unroll
            for (int d = 0; d < DL; ++d) acc[d] += __shfl_xor_sync(kFull, acc[d], off);
        }
        if (u != 0 || h >= (G <= 2 ? G : mt.nh)) return;
        if (mt.flags & kWhole) {
            const float inv = lt > 0.f ? p.v_scale / lt : 0.f;
            uint4* orow = reinterpret_cast<uint4*>(reinterpret_cast<TQ*>(p.out) + (size_t)(mt.obase + h) * D);
#pragma unroll
            for (int k = 0; k < CPL; ++k)
#pragma unroll
                for (int j = 0; j < QPC; ++j) {
                    float f[EPQ];
#pragma unroll
                    for (int e = 0; e < EPQ; ++e) f[e] = acc[k * EPC + j * EPQ + e] * inv;
                    orow[(c + Q * k) * QPC + j] = Elem<TQ>::narrow(f);
                }
        } else {
            const float vs = p.v_scale;
            float4* prow = reinterpret_cast<float4*>(p.part_acc + (size_t)(mt.pidx + h) * D);
#pragma unroll
            for (int k = 0; k < CPL; ++k)
#pragma unroll
                for (int e = 0; e < EPC; e += 4)
                    prow[((c + Q * k) * EPC + e) / 4] =
                        make_float4(acc[k * EPC + e] * vs, acc[k * EPC + e + 1] * vs,
                                    acc[k * EPC + e + 2] * vs, acc[k * EPC + e + 3] * vs);
            if (c == 0) p.part_ml[mt.pidx + h] = make_float2(m_run, lt);
        }
    }
};

// ===========================================================================
// Tensor-core consumer (mma.sync m16n8k16, fp32 accumulate) for 16-bit
// elements and G in {4, 8}.  Per 16-token slice of a block:
//   S^T[16 tok x 8 heads] = K[16 x D] . Q^T[D x 8]       (D/16 MMAs)
//   O^T[D x 8 heads]     += V^T[D x 16 tok] . P^T[16 x 8] (D/16 MMAs)
// Lane = (r = lane / 4, c = lane % 4).  The contraction index of an MMA may
// be any fixed permutation of the head dims (resp. tokens) as long as both
// operands use it, so every lane loads whole 16-byte chunks of the tile with
// plain shared loads:
//   QK step (j, hf): k-slots (2c, 2c+1) <-> dims 8(4j+c) + 4hf + {0,1},
//                    k-slots (2c+8, 2c+9) <-> dims 8(4j+c) + 4hf + {2,3};
//   PV tile m: row r <-> dim r*D/8 + 2m, row r+8 <-> dim r*D/8 + 2m + 1,
//              k-slot i <-> token i; V^T pairs of adjacent tokens are
//              assembled with byte permutes.
// P is rounded to the element type for the second MMA and the softmax sums
// use the rounded values.  Heads >= G of the 8 MMA columns are zero padding.
// ===========================================================================
template <typename T, int D, int BS, int G>
struct MmaConsumer {
    static constexpr bool kPairs = false;   // one block per consumer step
    using S = DecodeShape<T, T, D, BS, G>;
    static_assert(sizeof(T) == 2, "tensor-core consumer needs 16-bit elements");
    static_assert(G <= 8, "the 8 MMA columns hold the query heads of one group");
    static constexpr int KJ = D / 32;      // 16-byte chunks per lane per K row
    static constexpr int MT = D / 16;      // PV MMAs (row tiles of 16 dims)
    static constexpr int VCH = D / 64;     // 16-byte chunks per lane per V row (D/8 dims)
    static_assert(D % 64 == 0, "head_size 64 or 128");

    int r, c;
    uint32_t qf[KJ][4];                    // Q^T fragments (b0, b1 for hf = 0, 1)
    float o[MT][4];                        // O^T accumulators
    float m0, m1, l0, l1;                  // heads 2c, 2c+1

    __device__ __forceinline__ static void mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
        if constexpr (std::is_same<T, __nv_bfloat16>::value) {
            asm volatile(
                "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
                "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
        } else {
            asm volatile(
                "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, "
                "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
        }
    }

    __device__ __forceinline__ static uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
        uint32_t d;
        asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
        return d;
    }

    __device__ __forceinline__ static float lo_f(uint32_t w) {
        if constexpr (std::is_same<T, __nv_bfloat16>::value) return __uint_as_float(w << 16);
        else return __half2float(__ushort_as_half((unsigned short)(w & 0xffffu)));
    }
    __device__ __forceinline__ static float hi_f(uint32_t w) {
        if constexpr (std::is_same<T, __nv_bfloat16>::value) return __uint_as_float(w & 0xffff0000u);
        else return __half2float(__ushort_as_half((unsigned short)(w >> 16)));
    }

    __device__ __forceinline__ void init(int lane) {
        r = lane >> 2;
        c = lane & 3;
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
#pragma unroll
        for (int m = 0; m < MT; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;
#pragma unroll
        for (int j = 0; j < KJ; ++j) qf[j][0] = qf[j][1] = qf[j][2] = qf[j][3] = 0u;
    }

    __device__ __forceinline__ void begin(const unsigned char* qslot, float, int nh) {
        // B operand: column n = head r; rows = permuted dims of chunk 4j + c.
#pragma unroll
        for (int j = 0; j < KJ; ++j) {
            uint4 w = make_uint4(0u, 0u, 0u, 0u);
            if (r < nh) w = reinterpret_cast<const uint4*>(qslot + r * S::ROW)[4 * j + c];
            qf[j][0] = w.x;
            qf[j][1] = w.y;
            qf[j][2] = w.z;
            qf[j][3] = w.w;
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
    }

    __device__ __forceinline__ void slice(const unsigned char* Kt, const unsigned char* Vt,
                                          int nvalid, float scale_log2) {
        // ---- S^T = K . Q^T ----
        const uint4* k0 = reinterpret_cast<const uint4*>(Kt + r * S::ROW);
        const uint4* k8 = reinterpret_cast<const uint4*>(Kt + (r + 8) * S::ROW);
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < KJ; ++j) {
            const uint4 a = k0[4 * j + c];
            const uint4 b = k8[4 * j + c];
            mma(sc, a.x, b.x, a.y, b.y, qf[j][0], qf[j][1]);
            mma(sc, a.z, b.z, a.w, b.w, qf[j][2], qf[j][3]);
        }
        // sc: [tok r][head 2c], [tok r][2c+1], [tok r+8][2c], [tok r+8][2c+1]
        const bool v0 = r < nvalid, v8 = r + 8 < nvalid;
        const float z0 = v0 ? sc[0] * scale_log2 : -INFINITY;
        const float z1 = v0 ? sc[1] * scale_log2 : -INFINITY;
        const float z2 = v8 ? sc[2] * scale_log2 : -INFINITY;
        const float z3 = v8 ? sc[3] * scale_log2 : -INFINITY;
        float mx0 = fmaxf(z0, z2), mx1 = fmaxf(z1, z3);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, off));
        }
        const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);   // finite: nvalid > 0
        const float al0 = ex2(m0 - n0), al1 = ex2(m1 - n1);
        m0 = n0;
        m1 = n1;
        const uint32_t pk_lo = Elem<T>::pack2(ex2(z0 - n0), ex2(z1 - n1));   // token r
        const uint32_t pk_hi = Elem<T>::pack2(ex2(z2 - n0), ex2(z3 - n1));   // token r + 8
        l0 = l0 * al0 + lo_f(pk_lo) + lo_f(pk_hi);
        l1 = l1 * al1 + hi_f(pk_lo) + hi_f(pk_hi);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            o[m][0] *= al0;
            o[m][2] *= al0;
            o[m][1] *= al1;
            o[m][3] *= al1;
        }
        // ---- B = P^T: lane (r, c) needs P[head r][tokens 2c, 2c+1, 2c+8, 2c+9] ----
        const int src0 = (2 * c) * 4 + (r >> 1), src1 = src0 + 4;
        const uint32_t sel = (r & 1) ? 0x7632u : 0x5410u;
        const uint32_t x0 = __shfl_sync(kFull, pk_lo, src0), x1 = __shfl_sync(kFull, pk_lo, src1);
        const uint32_t y0 = __shfl_sync(kFull, pk_hi, src0), y1 = __shfl_sync(kFull, pk_hi, src1);
        const uint32_t pb0 = prmt(x0, x1, sel), pb1 = prmt(y0, y1, sel);
        // ---- O^T += V^T . P^T ----
        uint32_t w[4][4 * VCH];   // rows 2c, 2c+1, 2c+8, 2c+9; words = dim pairs
        const int rows[4] = {2 * c, 2 * c + 1, 2 * c + 8, 2 * c + 9};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4* vr = reinterpret_cast<const uint4*>(Vt + rows[i] * S::ROW) + r * VCH;
            const bool ok = rows[i] < nvalid;
#pragma unroll
            for (int ch = 0; ch < VCH; ++ch) {
                uint4 v = vr[ch];
                if (!ok) v = make_uint4(0u, 0u, 0u, 0u);   // masked tokens may hold NaN
                w[i][4 * ch + 0] = v.x;
                w[i][4 * ch + 1] = v.y;
                w[i][4 * ch + 2] = v.z;
                w[i][4 * ch + 3] = v.w;
            }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const uint32_t a0 = prmt(w[0][m], w[1][m], 0x5410u);
            const uint32_t a1 = prmt(w[0][m], w[1][m], 0x7632u);
            const uint32_t a2 = prmt(w[2][m], w[3][m], 0x5410u);
            const uint32_t a3 = prmt(w[2][m], w[3][m], 0x7632u);
            mma(o[m], a0, a1, a2, a3, pb0, pb1);
        }
    }

    __device__ __forceinline__ void block(const unsigned char* Kt, const unsigned char* Vt,
                                          int nvalid, float scale_log2) {
#pragma unroll
        for (int sl = 0; sl < BS / 16; ++sl) {
            const int nv = nvalid - 16 * sl;
            if (nv <= 0) break;
            slice(Kt + sl * 16 * S::ROW, Vt + sl * 16 * S::ROW, nv, scale_log2);
        }
    }

    __device__ __forceinline__ void finish(const StageMeta& mt, const DecodeParams& p) {
        float t0 = l0, t1 = l1;
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            t0 += __shfl_xor_sync(kFull, t0, off);
            t1 += __shfl_xor_sync(kFull, t1, off);
        }
        // lane (r, c) holds dims [r*D/8, (r+1)*D/8) of heads 2c, 2c+1
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int head = 2 * c + e;
            if (head >= (G <= 2 ? G : mt.nh)) continue;
            const float lt = e ? t1 : t0;
            if (mt.flags & kWhole) {
                const float inv = lt > 0.f ? p.v_scale / lt : 0.f;
                uint32_t words[MT];
#pragma unroll
                for (int m = 0; m < MT; ++m) words[m] = Elem<T>::pack2(o[m][e] * inv, o[m][2 + e] * inv);
                uint4* orow = reinterpret_cast<uint4*>(reinterpret_cast<T*>(p.out) +
                                                       (size_t)(mt.obase + head) * D + r * (D / 8));
#pragma unroll
                for (int ch = 0; ch < VCH; ++ch)
                    orow[ch] = make_uint4(words[4 * ch], words[4 * ch + 1], words[4 * ch + 2],
                                          words[4 * ch + 3]);
            } else {
                const float vs = p.v_scale;
                float4* prow = reinterpret_cast<float4*>(p.part_acc + (size_t)(mt.pidx + head) * D +
                                                         r * (D / 8));
#pragma unroll
                for (int m = 0; m < MT; m += 2)
                    prow[m / 2] = make_float4(o[m][e] * vs, o[m][2 + e] * vs, o[m + 1][e] * vs,
                                              o[m + 1][2 + e] * vs);
                if (r == 0)
                    p.part_ml[mt.pidx + head] = make_float2(e ? m1 : m0, lt);
            }
        }
    }
};

// ===========================================================================
// Tensor-core consumer for an FP8 (E4M3) cache and 16-bit q/out, G in {4, 8}.
// E4M3 converts exactly to fp16, so both products run as fp16 mma.m16n8k16
// (q is rounded to fp16 when it is bf16).  Fragment layout as in
// MmaConsumer, with 16 dims per 16-byte chunk of a cache row:
//   QK step (j, hf): k-slots (2c, 2c+1) <-> dims 16(4j+c) + 4hf + {0,1},
//                    k-slots (2c+8, 2c+9) <-> dims 16(4j+c) + 4hf + {2,3};
//   PV tile m: row r <-> dim r*D/8 + 2m, row r+8 <-> dim r*D/8 + 2m + 1;
// V^T pairs of adjacent tokens are gathered byte-wise with permutes, then
// converted pairwise.  The per-tensor scales enter the logits (k_scale) and
// the output (v_scale).
// ===========================================================================
template <typename TQ, int D, int BS, int G>
struct MmaConsumerFp8 {
    using S = DecodeShape<TQ, fp8e4m3, D, BS, G>;
    static_assert(sizeof(TQ) == 2, "q must be 16-bit");
    static_assert(G <= 8, "the 8 MMA columns hold the query heads of one group");
    static_assert(D % 64 == 0, "head_size 64 or 128");
    static constexpr int KJ = D / 64;      // 16-dim chunks per lane per K row
    static constexpr int MT = D / 16;      // PV MMAs
    static constexpr int VB = D / 8;       // V bytes (dims) per lane per row

    int r, c;
    uint32_t qf[KJ][8];                    // fp16 pairs: [hf][b0, b1] for hf = 0..3
    float o[MT][4];
    float m0, m1, l0, l1;

    __device__ __forceinline__ static void mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, "
            "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    }
    __device__ __forceinline__ static uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
        uint32_t d;
        asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
        return d;
    }
    __device__ __forceinline__ static uint32_t to_f16x2(uint32_t w) {
        if constexpr (std::is_same<TQ, __half>::value) {
            return w;
        } else {
            float lo, hi;
            Elem<__nv_bfloat16>::widen2(w, lo, hi);
            return Elem<__half>::pack2(lo, hi);
        }
    }
    __device__ __forceinline__ static float lo_f(uint32_t w) {
        return __half2float(__ushort_as_half((unsigned short)(w & 0xffffu)));
    }
    __device__ __forceinline__ static float hi_f(uint32_t w) {
        return __half2float(__ushort_as_half((unsigned short)(w >> 16)));
    }

    __device__ __forceinline__ void init(int lane) {
        r = lane >> 2;
        c = lane & 3;
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
#pragma unroll
        for (int m = 0; m < MT; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;
#pragma unroll
        for (int j = 0; j < KJ; ++j)
#pragma unroll
            for (int i = 0; i < 8; ++i) qf[j][i] = 0u;
    }

    __device__ __forceinline__ void begin(const unsigned char* qslot, float, int nh) {
#pragma unroll
        for (int j = 0; j < KJ; ++j) {
            uint4 a = make_uint4(0u, 0u, 0u, 0u), b = a;
            if (r < nh) {
                const uint4* qrow = reinterpret_cast<const uint4*>(qslot + r * S::QROW);
                a = qrow[2 * (4 * j + c)];          // dims 16(4j+c) + 0..7
                b = qrow[2 * (4 * j + c) + 1];      // dims 16(4j+c) + 8..15
            }
            const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) qf[j][i] = to_f16x2(w[i]);
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) o[m][0] = o[m][1] = o[m][2] = o[m][3] = 0.f;
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
    }

    // S^T of one 16-token slice: sc = K[16 x D] . Q^T (D/16 MMAs)
    __device__ __forceinline__ void qk(const unsigned char* Kt, float (&sc)[4]) const {
        const uint4* k0 = reinterpret_cast<const uint4*>(Kt + r * S::ROW);
        const uint4* k8 = reinterpret_cast<const uint4*>(Kt + (r + 8) * S::ROW);
#pragma unroll
        for (int j = 0; j < KJ; ++j) {
            const uint4 a = k0[4 * j + c];
            const uint4 b = k8[4 * j + c];
            const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int hf = 0; hf < 4; ++hf)
                mma(sc, e4m3x2_to_f16x2((uint16_t)(wa[hf] & 0xffffu)),
                    e4m3x2_to_f16x2((uint16_t)(wb[hf] & 0xffffu)),
                    e4m3x2_to_f16x2((uint16_t)(wa[hf] >> 16)), e4m3x2_to_f16x2((uint16_t)(wb[hf] >> 16)),
                    qf[j][2 * hf], qf[j][2 * hf + 1]);
        }
    }

    // Logits of a slice in log2 units; tokens at or past nvalid are -inf.
    __device__ __forceinline__ void logits(const float (&sc)[4], int nvalid, float scale_log2,
                                           float (&z)[4]) const {
        const bool v0 = r < nvalid, v8 = r + 8 < nvalid;
        z[0] = v0 ? sc[0] * scale_log2 : -INFINITY;
        z[1] = v0 ? sc[1] * scale_log2 : -INFINITY;
        z[2] = v8 ? sc[2] * scale_log2 : -INFINITY;
        z[3] = v8 ? sc[3] * scale_log2 : -INFINITY;
    }

    // Weights of a slice against the new maxima (fp16 pairs), added to l, and
    // moved to the B-fragment layout of the PV products.
    __device__ __forceinline__ void weights(const float (&z)[4], float n0, float n1, float& s0, float& s1,
                                            uint32_t& pb0, uint32_t& pb1) const {
        const uint32_t pk_lo = Elem<__half>::pack2(ex2(z[0] - n0), ex2(z[1] - n1));
        const uint32_t pk_hi = Elem<__half>::pack2(ex2(z[2] - n0), ex2(z[3] - n1));
        s0 += lo_f(pk_lo) + lo_f(pk_hi);
        s1 += hi_f(pk_lo) + hi_f(pk_hi);
        const int src0 = (2 * c) * 4 + (r >> 1), src1 = src0 + 4;
        const uint32_t sel = (r & 1) ? 0x7632u : 0x5410u;
        const uint32_t x0 = __shfl_sync(kFull, pk_lo, src0), x1 = __shfl_sync(kFull, pk_lo, src1);
        const uint32_t y0 = __shfl_sync(kFull, pk_hi, src0), y1 = __shfl_sync(kFull, pk_hi, src1);
        pb0 = prmt(x0, x1, sel);
        pb1 = prmt(y0, y1, sel);
    }

    // New running maxima from a slice's (or two slices') row maxima; rescales
    // l and the accumulator.  Returns the maxima to take weights against.
    __device__ __forceinline__ void update_max(float mx0, float mx1, float& n0, float& n1) {
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, off));
        }
        n0 = fmaxf(m0, mx0);
        n1 = fmaxf(m1, mx1);
        const float al0 = ex2(m0 - n0), al1 = ex2(m1 - n1);
        m0 = n0;
        m1 = n1;
        l0 *= al0;
        l1 *= al1;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            o[m][0] *= al0;
            o[m][2] *= al0;
            o[m][1] *= al1;
            o[m][3] *= al1;
        }
    }

    // O^T += V^T[D x 16 tok] . P^T (D/16 MMAs)
    __device__ __forceinline__ void pv(const unsigned char* Vt, int nvalid, uint32_t pb0, uint32_t pb1) {
        // V rows 2c, 2c+1, 2c+8, 2c+9: bytes = dims r*D/8 .. +D/8
        uint32_t w[4][VB / 4];
        const int rows[4] = {2 * c, 2 * c + 1, 2 * c + 8, 2 * c + 9};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const bool ok = rows[i] < nvalid;       // masked tokens may hold NaN codes
            const unsigned char* vr = Vt + rows[i] * S::ROW + r * VB;
            if constexpr (VB == 16) {
                uint4 v = *reinterpret_cast<const uint4*>(vr);
                if (!ok) v = make_uint4(0u, 0u, 0u, 0u);
                w[i][0] = v.x; w[i][1] = v.y; w[i][2] = v.z; w[i][3] = v.w;
            } else {
                uint2 v = *reinterpret_cast<const uint2*>(vr);
                if (!ok) v = make_uint2(0u, 0u);
                w[i][0] = v.x; w[i][1] = v.y;
            }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            // bytes 2m, 2m+1 of two rows: {A[2m], B[2m], A[2m+1], B[2m+1]}
            const int wi = m >> 1;
            const uint32_t sel2 = (m & 1) ? 0x7362u : 0x5140u;
            const uint32_t lo = prmt(w[0][wi], w[1][wi], sel2);
            const uint32_t hi = prmt(w[2][wi], w[3][wi], sel2);
            mma(o[m], e4m3x2_to_f16x2((uint16_t)(lo & 0xffffu)), e4m3x2_to_f16x2((uint16_t)(lo >> 16)),
                e4m3x2_to_f16x2((uint16_t)(hi & 0xffffu)), e4m3x2_to_f16x2((uint16_t)(hi >> 16)), pb0, pb1);
        }
    }

    __device__ __forceinline__ void slice(const unsigned char* Kt, const unsigned char* Vt,
                                          int nvalid, float scale_log2) {
        float sc[4] = {0.f, 0.f, 0.f, 0.f}, z[4];
        qk(Kt, sc);
        logits(sc, nvalid, scale_log2, z);
        float n0, n1;
        update_max(fmaxf(z[0], z[2]), fmaxf(z[1], z[3]), n0, n1);
        uint32_t pb0, pb1;
        weights(z, n0, n1, l0, l1, pb0, pb1);
        pv(Vt, nvalid, pb0, pb1);
    }

    // Two 16-token slices of one item with one softmax update: the two
    // independent QK and PV chains overlap, halving the per-token latency
    // of the warp.
    __device__ __forceinline__ void slice2(const unsigned char* Ka, const unsigned char* Va, int nva,
                                           const unsigned char* Kb, const unsigned char* Vb, int nvb,
                                           float scale_log2) {
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f}, za[4], zb[4];
        qk(Ka, sa);
        qk(Kb, sb);
        logits(sa, nva, scale_log2, za);
        logits(sb, nvb, scale_log2, zb);
        float n0, n1;
        update_max(fmaxf(fmaxf(za[0], za[2]), fmaxf(zb[0], zb[2])), fmaxf(fmaxf(za[1], za[3]), fmaxf(zb[1], zb[3])),
                   n0, n1);
        uint32_t pa0, pa1, pb0, pb1;
        weights(za, n0, n1, l0, l1, pa0, pa1);
        weights(zb, n0, n1, l0, l1, pb0, pb1);
        pv(Va, nva, pa0, pa1);
        pv(Vb, nvb, pb0, pb1);
    }

    // Pairs of blocks of one item are handed to block2 (block size 16: one
    // slice each); a 32-token block is a pair of slices itself.  With 8
    // query heads the MMA columns are full and the pair's extra registers
    // cost more than the overlap gains (measured), so G = 8 takes one slice
    // at a time.
    static constexpr bool kPairSlices = G < 8;
    static constexpr bool kPairs = BS == 16 && kPairSlices;

    __device__ __forceinline__ void block(const unsigned char* Kt, const unsigned char* Vt,
                                          int nvalid, float scale_log2) {
        if (BS == 32 && kPairSlices && nvalid > 16) {
            slice2(Kt, Vt, 16, Kt + 16 * S::ROW, Vt + 16 * S::ROW, nvalid - 16, scale_log2);
            return;
        }
#pragma unroll
        for (int sl = 0; sl < BS / 16; ++sl) {
            const int nv = nvalid - 16 * sl;
            if (nv <= 0) break;
            slice(Kt + sl * 16 * S::ROW, Vt + sl * 16 * S::ROW, nv, scale_log2);
        }
    }

    __device__ __forceinline__ void block2(const unsigned char* Ka, const unsigned char* Va, int nva,
                                           const unsigned char* Kb, const unsigned char* Vb, int nvb,
                                           float scale_log2) {
        slice2(Ka, Va, nva, Kb, Vb, nvb, scale_log2);
    }

    __device__ __forceinline__ void finish(const StageMeta& mt, const DecodeParams& p) {
        float t0 = l0, t1 = l1;
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            t0 += __shfl_xor_sync(kFull, t0, off);
            t1 += __shfl_xor_sync(kFull, t1, off);
        }
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int head = 2 * c + e;
            if (head >= (G <= 2 ? G : mt.nh)) continue;
            const float lt = e ? t1 : t0;
            if (mt.flags & kWhole) {
                const float inv = lt > 0.f ? p.v_scale / lt : 0.f;
                uint32_t words[MT];
#pragma unroll
                for (int m = 0; m < MT; ++m) words[m] = Elem<TQ>::pack2(o[m][e] * inv, o[m][2 + e] * inv);
                uint4* orow = reinterpret_cast<uint4*>(reinterpret_cast<TQ*>(p.out) +
                                                       (size_t)(mt.obase + head) * D + r * (D / 8));
#pragma unroll
                for (int ch = 0; ch < MT / 4; ++ch)
                    orow[ch] = make_uint4(words[4 * ch], words[4 * ch + 1], words[4 * ch + 2],
                                          words[4 * ch + 3]);
            } else {
                const float vs = p.v_scale;
                float4* prow = reinterpret_cast<float4*>(p.part_acc + (size_t)(mt.pidx + head) * D +
                                                         r * (D / 8));
#pragma unroll
                for (int m = 0; m < MT; m += 2)
                    prow[m / 2] = make_float4(o[m][e] * vs, o[m][2 + e] * vs, o[m + 1][e] * vs,
                                              o[m + 1][2 + e] * vs);
                if (r == 0)
                    p.part_ml[mt.pidx + head] = make_float2(e ? m1 : m0, lt);
            }
        }
    }
};

// Tensor cores where the fp32 FMA path is issue-bound: groups of 4-8 query
// heads over a 16-bit cache, and every group over an FP8 cache (half the
// bytes per element, so twice the FMA work per byte); columns of the 8-wide
// MMA beyond G are zero padding.
template <typename TQ, typename TC, int G>
struct UseMma {
    static constexpr bool value =
        sizeof(TQ) == 2 && ((std::is_same<TQ, TC>::value && (G == 4 || G == 8)) ||
                            (std::is_same<TC, fp8e4m3>::value && G <= 8));
};

template <typename TQ, typename TC, int D, int BS, int G>
using ConsumerFor = typename std::conditional<
    UseMma<TQ, TC, G>::value,
    typename std::conditional<std::is_same<TC, fp8e4m3>::value, MmaConsumerFp8<TQ, D, BS, G>,
                              MmaConsumer<TQ, D, BS, G>>::type,
    FmaConsumer<TQ, TC, D, BS, G>>::type;

// ===========================================================================
// Partition size for the call, chosen identically by every CTA.  With NW
// warps and n items of equal size the step lasts ceil(n / NW) item-times
// while the work is n / NW of them: a last round that is only partly full
// leaves warps idle.  Among the block multiples in [partition_min,
// partition_size], take the largest whose fill ratio (n/NW) / ceil(n/NW) is
// within 0.02 of the best.
// ===========================================================================
constexpr int kMaxPartitionCandidates = 49;

__device__ __forceinline__ int choose_partition(const int* s_len, int nseq, const DecodeParams& p,
                                                int bs) {
    __shared__ int s_count[kMaxPartitionCandidates];
    __shared__ int s_choice;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    const int nc = min((p.partition_size - p.partition_min) / bs + 1, kMaxPartitionCandidates);
    for (int j = warp; j < nc; j += nwarps) {
        const int ps = p.partition_size - j * bs;
        int n = 0;
        for (int i = lane; i < nseq; i += 32) n += max(1, (s_len[i] + ps - 1) / ps);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) n += __shfl_xor_sync(kFull, n, off);
        if (lane == 0) s_count[j] = n;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const float nw = (float)(gridDim.x * p.warps);
        auto fill = [&](int j) {
            const float x = (float)s_count[j] * p.num_kv_heads * p.slices / nw;
            return x / ceilf(x);
        };
        float best = 0.f;
        for (int j = 0; j < nc; ++j) best = fmaxf(best, fill(j));
        int pick = 0;
        while (fill(pick) < best - 0.02f) ++pick;
        s_choice = p.partition_size - pick * bs;
    }
    __syncthreads();
    return s_choice;
}

// ===========================================================================
// The kernel: prologue, producer (bulk-copy ring) and consumer loop.
// ===========================================================================
#ifndef PKV_FP8_THREADS
#define PKV_FP8_THREADS 512
#endif
// Up to 12 consumer warps (16 for the tensor-core consumer over an FP8
// cache, whose tiles are half the size) per CTA; the host picks the count.
template <typename TQ, typename TC, int G>
constexpr int decode_max_threads() {
    return (std::is_same<TC, fp8e4m3>::value && UseMma<TQ, TC, G>::value) ? PKV_FP8_THREADS : 384;
}

template <typename TQ, typename TC, int D, int BS, int G>
__global__ void __launch_bounds__(decode_max_threads<TQ, TC, G>(), 1) paged_decode_kernel(const DecodeParams p) {
    using S = DecodeShape<TQ, TC, D, BS, G>;
    using L = WarpSmem<TQ, TC, D, BS, G>;
    constexpr bool kSameType = std::is_same<TQ, TC>::value;   // fused cache write needs it
    extern __shared__ __align__(128) unsigned char smem[];

    const int nseq = p.num_seqs;
    int* s_len = reinterpret_cast<int*>(smem);   // [S]
    int* s_pre = s_len + nseq;                   // [S + 1]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int R = p.stages;
    unsigned char* wb = smem + p.seq_smem + (size_t)warp * p.warp_smem;
    unsigned char* ring = wb + L::ring(R);
    unsigned char* qbuf = wb + L::qbuf(R);
    unsigned char* nbuf = wb + L::nbuf(R);
    StageMeta* meta = reinterpret_cast<StageMeta*>(wb + L::meta(R));
    const uint32_t bar0 = smem_addr(wb + L::bars(R));
    int PS = p.partition_size;

    if (lane == 0)
        for (int st = 0; st < R; ++st) mbar_init(bar0 + 8 * st, 1);
    fence_mbar_init();
    griddep_wait();      // inputs may come from the previous kernel on the stream

    // ---- lengths and partition prefix sums (every CTA; CTA 0 publishes) ----
    for (int i = threadIdx.x; i < nseq; i += blockDim.x) {
        int len = p.context_lens[i];
        if (len < 0 || len > p.max_blocks_per_seq * BS || len > p.max_context_len) {
            flag_error(p.errors, PKV_DEVERR_CONTEXT);
            len = 0;
        }
        s_len[i] = len;
    }
    __syncthreads();
    if (p.partition_min > 0) PS = choose_partition(s_len, nseq, p, BS);
    if (warp == 0) {
        int carry = 0;
        for (int base = 0; base < nseq; base += 32) {
            const int i = base + lane;
            const int n = (i < nseq) ? max(1, (s_len[i] + PS - 1) / PS) : 0;
            int incl = n;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_up_sync(kFull, incl, off);
                if (lane >= off) incl += v;
            }
            if (i < nseq) s_pre[i] = carry + incl - n;
            carry += __shfl_sync(kFull, incl, 31);
        }
        if (lane == 0) s_pre[nseq] = carry;
    }
    __syncthreads();
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i <= nseq; i += blockDim.x) p.prefix_out[i] = s_pre[i];
    griddep_launch();    // the merge kernel may get resident; it waits for our completion

    const int Hkv = p.num_kv_heads;
    const int Gr = p.group;                      // real group size
    const int NSL = p.slices;
    const int NV = Hkv * NSL;                    // (KV head, slice) pairs per partition
    const int n_items = s_pre[nseq] * NV;
    const int NW = gridDim.x * p.warps;
    const int gw = blockIdx.x * p.warps + warp;
    // Items of more than 32 blocks (partitions up to 64 blocks) only for
    // 16-bit caches and groups of 4+ heads; elsewhere the host keeps
    // partitions at 32 blocks or less and this code is left out.
    constexpr bool kLongItems = !std::is_same<TC, fp8e4m3>::value && G >= 4;

    auto fetch = [&](int idx) -> Item {
        Item it;
        it.idx = idx;
        it.s = it.vg = it.jsp = it.tok0 = it.ntok = it.whole = it.tbl = 0;
        it.nblk = 0;
        it.slot = -1;
        if (idx >= n_items) return it;
        const int jsp = idx / NV;
        it.vg = idx - jsp * NV;
        it.jsp = jsp;
        int lo = 0, hi = nseq - 1;  // largest s with s_pre[s] <= jsp
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_pre[mid] <= jsp) lo = mid; else hi = mid - 1;
        }
        it.s = lo;
        it.whole = (s_pre[lo + 1] - s_pre[lo]) == 1;
        it.tok0 = (jsp - s_pre[lo]) * PS;
        it.ntok = min(s_len[lo] - it.tok0, PS);
        const int used = (it.ntok + BS - 1) / BS;
        it.nblk = max(used, 1);
        if (lane < used)
            it.tbl = __ldg(p.block_tables + (size_t)lo * p.max_blocks_per_seq + it.tok0 / BS + lane);
        if (kSameType && p.slot_mapping != nullptr && it.ntok > 0 && it.tok0 + it.ntok == s_len[lo])
            it.slot = __ldg(p.slot_mapping + lo);
        return it;
    };
    auto next_index = [&]() -> int {
        int v = 0;
        if (lane == 0) v = atomicAdd(p.sched, 1) + NW;
        return __shfl_sync(kFull, v, 0);
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
    const TC* kc = reinterpret_cast<const TC*>(p.k_cache);
    const TC* vc = reinterpret_cast<const TC*>(p.v_cache);
    const TQ* qg = reinterpret_cast<const TQ*>(p.q);

    auto issue = [&]() {
        if (P.idx >= n_items) return;
        const int st = issue_st;
        if constexpr (kLongItems) {
            if (pj > 0 && (pj & 31) == 0) {
                // the item's next 32 block ids (an item of more than 32 blocks)
                const int used = (P.ntok + BS - 1) / BS;
                if (pj + lane < used)
                    P.tbl = __ldg(p.block_tables + (size_t)P.s * p.max_blocks_per_seq + P.tok0 / BS + pj + lane);
            }
        }
        const int phys = __shfl_sync(kFull, P.tbl, pj & 31);
        int nvalid = min(max(P.ntok - pj * BS, 0), BS);
        const bool bad = nvalid > 0 && (phys < 0 || phys >= p.num_blocks);
        if (bad) nvalid = 0;
        const bool first = pj == 0, last = pj == P.nblk - 1;
        // Fused cache write: the last block of the item that ends the sequence
        // holds the new token at row newrow; its slot must be that position.
        int newrow = -1;
        if (last && P.slot >= 0 && nvalid > 0) {
            newrow = nvalid - 1;
            if (P.slot != (int64_t)phys * BS + newrow) newrow = -2;   // not the last position
        }
        if (lane == 0) {
            int g = P.vg, sl = 0;                    // KV head and head slice
            if (NSL > 1) {
                g = P.vg / NSL;
                sl = P.vg - g * NSL;
            }
            const int head0 = g * Gr + sl * G;       // first query head of the item
            StageMeta m;
            m.pidx = (int64_t)P.jsp * p.num_heads + head0;
            m.obase = (int64_t)P.s * p.num_heads + head0;
            m.slot = P.slot;
            m.g = g;
            m.nh = min(G, Gr - sl * G);
            m.nvalid = nvalid;
            m.flags = (first ? kFirst : 0) | (last ? kLast : 0) | (P.whole ? kWhole : 0) | (sl == 0 ? kStore : 0);
            m.qslot = qslot_ctr;
            m.newrow = newrow < 0 ? -1 : newrow;
            meta[st] = m;
            const uint32_t bar = bar0 + 8 * st;
            const uint32_t qbytes = (uint32_t)m.nh * S::QROW;
            const uint32_t bytes = (first ? qbytes : 0) + (nvalid > 0 ? 2 * S::TILE : 0) +
                                   (newrow >= 0 ? 2 * S::ROW : 0);
            mbar_arrive_expect_tx(bar, bytes);
            if (newrow >= 0) {
                const TC* kn = reinterpret_cast<const TC*>(p.key) + (size_t)P.s * p.key_stride + (size_t)g * D;
                const TC* vn = reinterpret_cast<const TC*>(p.value) + (size_t)P.s * p.value_stride + (size_t)g * D;
                bulk_g2s(smem_addr(nbuf + (size_t)st * 2 * S::ROW), kn, S::ROW, bar);
                bulk_g2s(smem_addr(nbuf + (size_t)st * 2 * S::ROW + S::ROW), vn, S::ROW, bar);
            }
            if (newrow == -2) flag_error(p.errors, PKV_DEVERR_SLOT);
            if (first)
                bulk_g2s(smem_addr(qbuf + qslot_ctr * S::QBYTES), qg + (size_t)m.obase * D, qbytes, bar);
            if (nvalid > 0) {
                const size_t off = ((size_t)phys * Hkv + g) * tile_elems;
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

    // ---- consumer ----
    ConsumerFor<TQ, TC, D, BS, G> cons;
    const float qscale = p.scale_log2 * p.k_scale;   // logits in log2 units, cache scale folded in
    cons.init(lane);

    for (int i = 0; i < R; ++i) issue();
    int cons_st = 0;
    uint32_t phase = 0;
    int consumed = 0;
    bool lost = false;
    // A stage's copies have landed, as seen by every lane; false (for the whole
    // warp) once the wait gives up.
    auto stage_ready = [&](uint32_t bar, uint32_t parity) -> bool {
        return __all_sync(kFull, mbar_wait_bounded(bar, parity, p.wait_limit));
    };

    while (consumed < issued) {
        const uint32_t bar = bar0 + 8 * cons_st;
        if (!stage_ready(bar, phase)) {
            flag_error(p.errors, PKV_DEVERR_WAIT);
            lost = true;
            break;
        }
        // Over an FP8 cache (threads capped at 128 registers) only what the block
        // needs is held in registers and finish() reads the item's output rows
        // from the stage's metadata; the 16-bit kernels keep a copy (measured:
        // each way is the faster one for its kernel).
        constexpr bool kLean = std::is_same<TC, fp8e4m3>::value;
        StageMeta mt;
        if constexpr (kLean) {
            mt.flags = meta[cons_st].flags;
            mt.nvalid = meta[cons_st].nvalid;
            mt.newrow = meta[cons_st].newrow;
        } else {
            mt = meta[cons_st];
        }
        // (a column count of 1 or 2 only ever holds a whole group of that size)
        if (mt.flags & kFirst) cons.begin(qbuf + meta[cons_st].qslot * S::QBYTES, qscale, G <= 2 ? G : meta[cons_st].nh);
        using Cons = ConsumerFor<TQ, TC, D, BS, G>;
        if constexpr (Cons::kPairs) {
            // the item's next block is in the next stage: take both together
            if (!(mt.flags & kLast) && mt.nvalid > 0 && mt.newrow < 0 && consumed + 1 < issued) {
                const int st2 = (cons_st + 1 == R) ? 0 : cons_st + 1;
                const uint32_t ph2 = (cons_st + 1 == R) ? (phase ^ 1u) : phase;
                if (!stage_ready(bar0 + 8 * st2, ph2)) {
                    flag_error(p.errors, PKV_DEVERR_WAIT);
                    lost = true;
                    break;
                }
                const int nvalid2 = meta[st2].nvalid;
                if (nvalid2 > 0 && meta[st2].newrow < 0) {
                    const unsigned char* Ka = ring + (size_t)cons_st * 2 * S::TILE;
                    const unsigned char* Kb = ring + (size_t)st2 * 2 * S::TILE;
                    cons.block2(Ka, Ka + S::TILE, mt.nvalid, Kb, Kb + S::TILE, nvalid2, qscale);
                    if (meta[st2].flags & kLast) cons.finish(meta[st2], p);
                    __syncwarp();
                    consumed += 2;
                    cons_st = st2;
                    phase = ph2;
                    if (++cons_st == R) { cons_st = 0; phase ^= 1u; }
                    issue();
                    issue();
                    continue;
                }
            }
        }
        if (mt.newrow >= 0) {
            // Fused cache write: put the new token's K and V rows into the tile
            // (it holds the slot's old bytes) and into the cache slot.
            unsigned char* Kt = ring + (size_t)cons_st * 2 * S::TILE;
            const unsigned char* nb = nbuf + (size_t)cons_st * 2 * S::ROW;
            const int64_t slot = meta[cons_st].slot;
            const size_t slot_off = (size_t)slot / BS * Hkv * tile_elems +
                                    (size_t)meta[cons_st].g * tile_elems + (size_t)(slot % BS) * D;
            for (int ch = lane; ch < 2 * S::ROW / 16; ch += 32) {
                const int v = ch >= S::ROW / 16;
                const int c16 = ch - v * (S::ROW / 16);
                const uint4 w = reinterpret_cast<const uint4*>(nb + v * S::ROW)[c16];
                reinterpret_cast<uint4*>(Kt + v * S::TILE + mt.newrow * S::ROW)[c16] = w;
                if (meta[cons_st].flags & kStore) {
                    TC* cache = const_cast<TC*>(v ? vc : kc);
                    reinterpret_cast<uint4*>(cache + slot_off)[c16] = w;
                }
            }
            fence_proxy_async();     // these generic writes precede the stage's next bulk copy
            __syncwarp();
        }
        if (mt.nvalid > 0) {
            const unsigned char* Kt = ring + (size_t)cons_st * 2 * S::TILE;
            cons.block(Kt, Kt + S::TILE, mt.nvalid, qscale);
        }
        if (mt.flags & kLast) {
            if constexpr (kLean) cons.finish(meta[cons_st], p);
            else cons.finish(mt, p);
        }
        __syncwarp();
        ++consumed;
        if (++cons_st == R) { cons_st = 0; phase ^= 1u; }
        issue();
    }

    if (lost) {
        // Gave up: the copies already issued into this warp's stages still land
        // before the warp leaves (the CTA's shared memory must outlive them).
        int st = cons_st;
        uint32_t ph = phase;
        for (int k = consumed; k < issued; ++k) {
            mbar_wait_bounded(bar0 + 8 * st, ph, kWaitLimit);
            if (++st == R) { st = 0; ph ^= 1u; }
        }
        __syncwarp();
    }

    // Retire, on every path: the last warp to finish resets the scheduling
    // counters, so the next call on this workspace starts from zero.
    if (lane == 0) {
        __threadfence();
        const int done = atomicAdd(p.sched + 1, 1);
        if (done == NW - 1) {
            atomicExch(p.sched, 0);
            atomicExch(p.sched + 1, 0);
        }
    }
}

}  // namespace pkv
