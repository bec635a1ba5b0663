/*
 * CPU oracle for the paged KV-cache decode hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file.  Only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header or constant with the CUDA
 * library: the two meet only through the seeded inputs both are given.
 *
 * Everything here is the plain definition, in fp64, one (sequence, head)
 * row at a time, with no blocking, fusion or reordering.
 *
 * Sources (page titles as given on each page):
 *  [P5] "Efficient Memory Management for Large Language Model Serving with
 *       PagedAttention" summary page (xasun.com article 3997), section 2:
 *       attention keys/values live in non-contiguous fixed-size blocks that
 *       the kernel fetches block by block through a block table; section 1:
 *       reference counts plus copy-on-write share blocks between parallel
 *       samples and shared prefixes; the method leaves the output
 *       distribution unchanged (it is exact attention).
 *  [P1] "PyTorch-CUDA-v2.9 image enables PagedAttention" page (jsqmd.com
 *       164355), section on PagedAttention: the page table maps a logical
 *       position to a physical page of 16 tokens; decoding appends each new
 *       token's key/value; workflow list: prefill writes token KV into pages.
 *  [P4] "GPT-OSS memory management: PagedAttention explained" page
 *       (yongjin360.com 448593), section 2.2: a logical-to-physical table
 *       tells where token N's KV lives.
 *  [P2] "PagedAttention: accelerating GPT inference" page (yunthe.com
 *       621750), section 1.1: the attention is scaled dot-product attention.
 *
 * Readings the pages leave open (each taken as the plainest one):
 *  - the attention is softmax(scale * q.K^T) V over all cached tokens of the
 *    sequence, with no mask, bias or position term;
 *  - cache layout [num_blocks][num_kv_heads][block_size][head_size], the
 *    same for K and V; token t of a sequence sits in physical block
 *    block_table[t / block_size] at offset t % block_size;
 *  - query head h reads KV head h / (num_heads / num_kv_heads) (contiguous
 *    groups);
 *  - a sequence with context length 0 has an all-zero output.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F32 0
#define ORC_F16 1
#define ORC_BF16 2
#define ORC_E4M3 3   /* cache elements only: FP8 E4M3 times a per-tensor scale */

/* ---------------------------------------------------------------------
 * Element decoding: exact widening of the stored formats to fp64.
 * IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits.
 * bfloat16: the upper 16 bits of an IEEE binary32.
 * ------------------------------------------------------------------- */
static double orc_f16_to_double(uint16_t bits) {
    int sign = bits >> 15;
    int expo = (bits >> 10) & 0x1f;
    int frac = bits & 0x3ff;
    double v;
    if (expo == 0)
        v = ldexp((double)frac, -24);                 /* subnormal: frac * 2^-24 */
    else if (expo == 31)
        v = frac ? NAN : INFINITY;
    else
        v = ldexp((double)(frac | 0x400), expo - 25); /* 1.frac * 2^(expo-15) */
    return sign ? -v : v;
}

static double orc_bf16_to_double(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* FP8 E4M3 (the OCP 8-bit floating-point format): 1 sign bit, 4 exponent
 * bits with bias 7, 3 fraction bits; exponent field 0 holds subnormals
 * (fraction * 2^-9); there is no infinity and S.1111.111 is NaN; the largest
 * finite magnitude is 1.75 * 2^8 = 448. */
double orc_e4m3_to_double(uint8_t bits) {
    int sign = bits >> 7;
    int expo = (bits >> 3) & 0xf;
    int frac = bits & 0x7;
    double v;
    if (expo == 0xf && frac == 0x7)
        return NAN;
    if (expo == 0)
        v = ldexp((double)frac, -9);
    else
        v = ldexp((double)(frac | 0x8), expo - 10);  /* 1.frac * 2^(expo-7) */
    return sign ? -v : v;
}

/* Round to E4M3, nearest with ties to even, saturating: a magnitude that
 * would round above 448 becomes 448; NaN stays NaN (0x7f). */
uint8_t orc_double_to_e4m3(double x) {
    if (isnan(x)) return 0x7f;
    uint8_t sign = signbit(x) ? 0x80 : 0;
    double a = fabs(x);
    if (a >= 448.0) return sign | 0x7e;
    if (a == 0.0) return sign;
    int e2;
    frexp(a, &e2);
    int E = e2 - 1;
    if (E < -6) E = -6;                              /* subnormal range */
    double quantum = ldexp(1.0, E - 3);
    double r = nearbyint(a / quantum);
    long bits = ((long)(E + 7) << 3) + (long)r - 8;  /* carries into the next binade */
    if (bits > 0x7e) bits = 0x7e;                    /* 448 < a rounds up past 448 */
    return sign | (uint8_t)bits;
}

double orc_load(const void* base, int dtype, int64_t index) {
    if (dtype == ORC_F32) return (double)((const float*)base)[index];
    if (dtype == ORC_F16) return orc_f16_to_double(((const uint16_t*)base)[index]);
    return orc_bf16_to_double(((const uint16_t*)base)[index]);
}

/* ---------------------------------------------------------------------
 * Rounding fp64 -> storage format, round to nearest, ties to even, in one
 * step (no intermediate fp32).  For a format with p significand bits,
 * minimum normal exponent emin and exponent bias B, a finite |x| is
 * quantised to a multiple of 2^(E - (p-1)), E = max(floor(log2|x|), emin);
 * the integer multiple r then encodes as ((E + B) << (p-1)) + r - 2^(p-1),
 * which also covers subnormals (E = emin, r < 2^(p-1)) and a carry into
 * the next binade (r = 2^p).
 * ------------------------------------------------------------------- */
static uint16_t orc_round_small(double x, int p, int emin, int bias, double overflow_at,
                                uint16_t inf_bits, uint16_t nan_bits) {
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    if (isnan(x)) return nan_bits;
    double a = fabs(x);
    if (a >= overflow_at) return sign | inf_bits;
    if (a == 0.0) return sign;
    int e2;
    frexp(a, &e2);          /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;         /* floor(log2 a) */
    if (E < emin) E = emin;
    double quantum = ldexp(1.0, E - (p - 1));
    double r = nearbyint(a / quantum); /* a / quantum is exact; default mode is RNE */
    long bits = ((long)(E + bias) << (p - 1)) + (long)r - (1L << (p - 1));
    return sign | (uint16_t)bits;
}

uint16_t orc_double_to_f16(double x) {
    /* max finite 65504 = (2 - 2^-10) * 2^15; halfway to 2^16 is 65520 */
    return orc_round_small(x, 11, -14, 15, 65520.0, 0x7c00, 0x7e00);
}

uint16_t orc_double_to_bf16(double x) {
    /* max finite (2 - 2^-7) * 2^127; halfway to 2^128 is (2 - 2^-8) * 2^127 */
    return orc_round_small(x, 8, -126, 127, ldexp(2.0 - ldexp(1.0, -8), 127), 0x7f80, 0x7fc0);
}

/* Round n fp64 values to the storage format (fp32 via the C conversion,
 * which rounds to nearest even). */
void orc_round(const double* in, void* out, int dtype, int64_t n) {
    for (int64_t i = 0; i < n; ++i) {
        if (dtype == ORC_F32)
            ((float*)out)[i] = (float)in[i];
        else if (dtype == ORC_F16)
            ((uint16_t*)out)[i] = orc_double_to_f16(in[i]);
        else
            ((uint16_t*)out)[i] = orc_double_to_bf16(in[i]);
    }
}

/* ---------------------------------------------------------------------
 * Page-table address of one cache element [P5 s.2; P1; P4 s.2.2]:
 * token t of a sequence lives in physical block table[t / bs], slot t % bs.
 * ------------------------------------------------------------------- */
static int64_t orc_cache_index(const int32_t* table_row, int t, int kv_head, int d,
                               int num_kv_heads, int block_size, int head_size) {
    int64_t phys = table_row[t / block_size];
    int64_t off = t % block_size;
    return ((phys * num_kv_heads + kv_head) * block_size + off) * head_size + d;
}

/* Gather the K and V rows of tokens [t0, t1) of one sequence and KV head
 * into contiguous fp64 arrays [t1 - t0][head_size]. */
/* A cache element's real value: the stored element, or for E4M3 the stored
 * code times the tensor's scale (exact in fp64). */
static double orc_cache_value(const void* cache, int cdtype, int64_t idx, double cscale) {
    if (cdtype == ORC_E4M3) return orc_e4m3_to_double(((const uint8_t*)cache)[idx]) * cscale;
    return orc_load(cache, cdtype, idx);
}

static void orc_gather(double* K, double* V, const void* k_cache, const void* v_cache, int cdtype,
                       double k_scale, double v_scale, const int32_t* table_row, int t0, int t1,
                       int kv_head, int num_kv_heads, int block_size, int head_size) {
    for (int t = t0; t < t1; ++t)
        for (int d = 0; d < head_size; ++d) {
            int64_t idx = orc_cache_index(table_row, t, kv_head, d, num_kv_heads, block_size, head_size);
            K[(int64_t)(t - t0) * head_size + d] = orc_cache_value(k_cache, cdtype, idx, k_scale);
            V[(int64_t)(t - t0) * head_size + d] = orc_cache_value(v_cache, cdtype, idx, v_scale);
        }
}

/* ---------------------------------------------------------------------
 * Softmax statistics of one query row over tokens [t0, t1) [P2 s.1.1]:
 *   z_t = scale * sum_d q_d K_td
 *   m   = max_t z_t
 *   l   = sum_t exp(z_t - m)
 *   acc = sum_t exp(z_t - m) V_t        (not divided by l)
 *   w_t = exp(z_t - m) / l              (the attention weights)
 * For an empty range m = -inf, l = 0, acc = 0.
 * ------------------------------------------------------------------- */
static void orc_row(double* acc, double* m_out, double* l_out, double* weights,
                    const void* q, int qdtype, const void* k_cache, const void* v_cache, int cdtype,
                    double k_scale, double v_scale, const int32_t* table_row, int t0, int t1,
                    int64_t qrow, int h, int num_heads, int num_kv_heads, int head_size, int block_size,
                    double scale) {
    int G = num_heads / num_kv_heads;
    int kv_head = h / G;
    int n = t1 - t0;
    for (int d = 0; d < head_size; ++d) acc[d] = 0.0;
    *m_out = -INFINITY;
    *l_out = 0.0;
    if (n <= 0) return;

    double* K = (double*)malloc(sizeof(double) * (size_t)n * head_size);
    double* V = (double*)malloc(sizeof(double) * (size_t)n * head_size);
    double* z = (double*)malloc(sizeof(double) * (size_t)n);
    double* qd = (double*)malloc(sizeof(double) * (size_t)head_size);
    orc_gather(K, V, k_cache, v_cache, cdtype, k_scale, v_scale, table_row, t0, t1, kv_head,
               num_kv_heads, block_size, head_size);
    for (int d = 0; d < head_size; ++d)
        qd[d] = orc_load(q, qdtype, (qrow * num_heads + h) * head_size + d);

    double m = -INFINITY;
    for (int t = 0; t < n; ++t) {
        double dot = 0.0;
        for (int d = 0; d < head_size; ++d) dot += qd[d] * K[(int64_t)t * head_size + d];
        z[t] = scale * dot;
        if (z[t] > m) m = z[t];
    }
    double l = 0.0;
    for (int t = 0; t < n; ++t) {
        double e = exp(z[t] - m);
        l += e;
        for (int d = 0; d < head_size; ++d) acc[d] += e * V[(int64_t)t * head_size + d];
    }
    if (weights)
        for (int t = 0; t < n; ++t) weights[t] = exp(z[t] - m) / l;
    *m_out = m;
    *l_out = l;
    free(K);
    free(V);
    free(z);
    free(qd);
}

/* ---------------------------------------------------------------------
 * Paged decode attention, one query token per sequence [P5 s.2]:
 *   out[s, h, :] = sum_t softmax_t(scale * q[s,h] . K_s[t]) V_s[t],
 * K_s, V_s gathered through block_tables[s] for t < context_lens[s].
 * q: [S, H, D]; caches: [NB, Hkv, bs, D]; out: fp64 [S, H, D].
 * Rows are independent, so they are spread over nthreads OpenMP threads.
 * ------------------------------------------------------------------- */
void orc_paged_attention_ex(double* out, const void* q, int qdtype, const void* k_cache,
                            const void* v_cache, int cdtype, double k_scale, double v_scale,
                            const int32_t* block_tables, int max_blocks_per_seq,
                            const int32_t* context_lens, int num_seqs, int num_heads,
                            int num_kv_heads, int head_size, int block_size, double scale,
                            int nthreads) {
    int64_t rows = (int64_t)num_seqs * num_heads;
#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        int s = (int)(r / num_heads), h = (int)(r % num_heads);
        double m, l;
        double* o = out + r * head_size;
        orc_row(o, &m, &l, NULL, q, qdtype, k_cache, v_cache, cdtype, k_scale, v_scale,
                block_tables + (int64_t)s * max_blocks_per_seq, 0, context_lens[s], s, h,
                num_heads, num_kv_heads, head_size, block_size, scale);
        for (int d = 0; d < head_size; ++d) o[d] = (l > 0.0) ? o[d] / l : 0.0;
    }
}

void orc_paged_attention(double* out, const void* q, const void* k_cache, const void* v_cache,
                         int dtype, const int32_t* block_tables, int max_blocks_per_seq,
                         const int32_t* context_lens, int num_seqs, int num_heads,
                         int num_kv_heads, int head_size, int block_size, double scale,
                         int nthreads) {
    orc_paged_attention_ex(out, q, dtype, k_cache, v_cache, dtype, 1.0, 1.0, block_tables,
                           max_blocks_per_seq, context_lens, num_seqs, num_heads, num_kv_heads,
                           head_size, block_size, scale, nthreads);
}

/* Attention weights of one (s, h) row: weights[t] for t < context_lens[s]. */
void orc_attention_weights(double* weights, const void* q, const void* k_cache,
                           const void* v_cache, int dtype, const int32_t* block_tables,
                           int max_blocks_per_seq, const int32_t* context_lens, int s, int h,
                           int num_heads, int num_kv_heads, int head_size, int block_size,
                           double scale) {
    double m, l;
    double* acc = (double*)malloc(sizeof(double) * (size_t)head_size);
    orc_row(acc, &m, &l, weights, q, dtype, k_cache, v_cache, dtype, 1.0, 1.0,
            block_tables + (int64_t)s * max_blocks_per_seq, 0, context_lens[s], s, h, num_heads,
            num_kv_heads, head_size, block_size, scale);
    free(acc);
}

/* ---------------------------------------------------------------------
 * Split-context statistics: for every (s, h) and partition p covering
 * tokens [p*ps, min(L, (p+1)*ps)), the unnormalised acc, m and l defined
 * in orc_row.  acc: [S, H, P, D], m and l: [S, H, P]; partitions past the
 * end of a sequence hold m = -inf, l = 0, acc = 0.
 * ------------------------------------------------------------------- */
void orc_partition_stats(double* acc, double* m, double* l, const void* q, const void* k_cache,
                         const void* v_cache, int dtype, const int32_t* block_tables,
                         int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
                         int num_heads, int num_kv_heads, int head_size, int block_size,
                         double scale, int partition_size, int num_partitions, int nthreads) {
    int64_t rows = (int64_t)num_seqs * num_heads * num_partitions;
#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
        int p = (int)(r % num_partitions);
        int64_t sh = r / num_partitions;
        int s = (int)(sh / num_heads), h = (int)(sh % num_heads);
        int L = context_lens[s];
        int t0 = p * partition_size;
        int t1 = t0 + partition_size < L ? t0 + partition_size : L;
        orc_row(acc + r * head_size, m + r, l + r, NULL, q, dtype, k_cache, v_cache, dtype, 1.0, 1.0,
                block_tables + (int64_t)s * max_blocks_per_seq, t0, t1, s, h, num_heads,
                num_kv_heads, head_size, block_size, scale);
    }
}

/* ---------------------------------------------------------------------
 * Log-sum-exp merge of partition statistics (the exact identity
 * softmax over a union = weighted combination of the parts):
 *   M = max_p m_p,  w_p = exp(m_p - M),
 *   out = sum_p w_p acc_p / sum_p w_p l_p.
 * acc: [R, P, D], m, l: [R, P]; out: [R, D].  All-empty rows give 0.
 * ------------------------------------------------------------------- */
void orc_lse_merge(double* out, const double* acc, const double* m, const double* l,
                   int64_t rows, int num_partitions, int head_size) {
    for (int64_t r = 0; r < rows; ++r) {
        double M = -INFINITY;
        for (int p = 0; p < num_partitions; ++p)
            if (m[r * num_partitions + p] > M) M = m[r * num_partitions + p];
        double den = 0.0;
        for (int d = 0; d < head_size; ++d) out[r * head_size + d] = 0.0;
        if (M == -INFINITY) continue;
        for (int p = 0; p < num_partitions; ++p) {
            double mp = m[r * num_partitions + p];
            if (mp == -INFINITY) continue;
            double w = exp(mp - M);
            den += w * l[r * num_partitions + p];
            for (int d = 0; d < head_size; ++d)
                out[r * head_size + d] += w * acc[(r * num_partitions + p) * head_size + d];
        }
        for (int d = 0; d < head_size; ++d) out[r * head_size + d] /= den;
    }
}

/* ---------------------------------------------------------------------
 * Cache write [P1 workflow; P5 s.2]: token i's K and V rows go to slot
 * slot_mapping[i] (block slot / bs, offset slot % bs) for every KV head;
 * a negative slot means "no write".  A byte copy: nothing is converted.
 * k, v: [T][...] with key_stride / value_stride elements between tokens and
 * head_size elements between heads.
 * ------------------------------------------------------------------- */
void orc_reshape_and_cache(const void* k, const void* v, void* k_cache, void* v_cache,
                           const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                           int head_size, int block_size, int elem_bytes, int64_t key_stride,
                           int64_t value_stride) {
    size_t row = (size_t)head_size * elem_bytes;
    for (int i = 0; i < num_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0) continue;
        int64_t b = slot / block_size, off = slot % block_size;
        for (int g = 0; g < num_kv_heads; ++g) {
            int64_t dst = ((b * num_kv_heads + g) * block_size + off) * head_size;
            memcpy((char*)k_cache + dst * elem_bytes,
                   (const char*)k + ((int64_t)i * key_stride + (int64_t)g * head_size) * elem_bytes, row);
            memcpy((char*)v_cache + dst * elem_bytes,
                   (const char*)v + ((int64_t)i * value_stride + (int64_t)g * head_size) * elem_bytes, row);
        }
    }
}

/* ---------------------------------------------------------------------
 * Copy-on-write block copy [P5 s.1, s.2]: for every layer and every pair
 * (src, dst) of block_mapping [N][2], physical block dst of that layer's
 * cache becomes a copy of block src.  Pairs are applied in order.
 * caches: array of num_layers host pointers, each [NB][block_bytes].
 * ------------------------------------------------------------------- */
void orc_copy_blocks(void** caches, int num_layers, const int64_t* block_mapping, int num_pairs,
                     int64_t block_bytes) {
    for (int layer = 0; layer < num_layers; ++layer)
        for (int i = 0; i < num_pairs; ++i) {
            int64_t src = block_mapping[2 * i], dst = block_mapping[2 * i + 1];
            memcpy((char*)caches[layer] + dst * block_bytes,
                   (const char*)caches[layer] + src * block_bytes, (size_t)block_bytes);
        }
}

/* ---------------------------------------------------------------------------
 * Swap between two block pools [P5 s.2: a block pool in GPU memory and one
 * in CPU memory, the latter for swapping; recovery by swap]: for every cache
 * c and pair i, block dst of dst_pools[c] becomes a copy of block src of
 * src_pools[c].  Pairs are applied in order.
 * ------------------------------------------------------------------- */
void orc_swap_blocks(void** src_pools, void** dst_pools, int num_caches, const int64_t* mapping,
                     int num_pairs, int64_t block_bytes) {
    for (int c = 0; c < num_caches; ++c)
        for (int i = 0; i < num_pairs; ++i)
            memcpy((char*)dst_pools[c] + mapping[2 * i + 1] * block_bytes,
                   (const char*)src_pools[c] + mapping[2 * i] * block_bytes, (size_t)block_bytes);
}

/* ---------------------------------------------------------------------------
 * Cache write into an E4M3 cache: code = e4m3(fp32(x) / fp32(scale)), the
 * quotient correctly rounded in fp32 (the precision the kernel takes the
 * decision in), then rounded to E4M3 as orc_double_to_e4m3 does.
 * k, v: [T][...] in src_dtype with key_stride / value_stride elements between
 * tokens; caches: uint8 [NB][Hkv][bs][D].
 * ------------------------------------------------------------------- */
uint8_t orc_quantize_e4m3(double x, float scale) {
    float q = (float)x / scale;          /* x is exact in fp32 for every source format */
    return orc_double_to_e4m3((double)q);
}

void orc_reshape_and_cache_e4m3(const void* k, const void* v, int src_dtype, uint8_t* k_cache,
                                uint8_t* v_cache, const int64_t* slot_mapping, int num_tokens,
                                int num_kv_heads, int head_size, int block_size,
                                int64_t key_stride, int64_t value_stride, float k_scale,
                                float v_scale) {
    for (int i = 0; i < num_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0) continue;
        int64_t b = slot / block_size, off = slot % block_size;
        for (int g = 0; g < num_kv_heads; ++g)
            for (int d = 0; d < head_size; ++d) {
                int64_t dst = ((b * num_kv_heads + g) * block_size + off) * head_size + d;
                k_cache[dst] = orc_quantize_e4m3(
                    orc_load(k, src_dtype, (int64_t)i * key_stride + (int64_t)g * head_size + d), k_scale);
                v_cache[dst] = orc_quantize_e4m3(
                    orc_load(v, src_dtype, (int64_t)i * value_stride + (int64_t)g * head_size + d), v_scale);
            }
    }
}

/* ---------------------------------------------------------------------------
 * Paged prefill / chunked-prefill attention [P1 workflow: prefill writes the
 * input tokens' KV into pages and decoding continues from them; P1 usage:
 * enable_chunked_prefill].  Sequence s holds context_lens[s] = L tokens in
 * its blocks, the last n = qsl[s+1] - qsl[s] of which are this call's
 * queries, packed as q rows qsl[s] .. qsl[s+1]-1.  Query i sits at position
 * L - n + i and attends causally to keys 0 .. L - n + i:
 *   out[qsl[s]+i, h, :] = sum_{t <= L-n+i} softmax_t(scale q.K_s[t]) V_s[t].
 * q, out: [T][H][D] with T = qsl[S]; out in fp64.
 * ------------------------------------------------------------------- */
void orc_paged_prefill(double* out, const void* q, const void* k_cache, const void* v_cache,
                       int dtype, const int32_t* block_tables, int max_blocks_per_seq,
                       const int32_t* context_lens, const int32_t* query_start_loc, int num_seqs,
                       int num_heads, int num_kv_heads, int head_size, int block_size, double scale,
                       int nthreads) {
    int64_t T = query_start_loc[num_seqs];
    int64_t rows = T * num_heads;
#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 4)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t row = r / num_heads;
        int h = (int)(r % num_heads);
        int s = 0;
        while (query_start_loc[s + 1] <= row) ++s;
        int n = query_start_loc[s + 1] - query_start_loc[s];
        int L = context_lens[s];
        int pos = L - n + (int)(row - query_start_loc[s]);
        double m, l;
        double* o = out + r * head_size;
        orc_row(o, &m, &l, NULL, q, dtype, k_cache, v_cache, dtype, 1.0, 1.0,
                block_tables + (int64_t)s * max_blocks_per_seq, 0, pos + 1, row, h, num_heads,
                num_kv_heads, head_size, block_size, scale);
        for (int d = 0; d < head_size; ++d) o[d] = (l > 0.0) ? o[d] / l : 0.0;
    }
}
