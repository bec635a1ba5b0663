/*
 * pagedkv.h -- C ABI of the B200 (sm_100a) paged KV-cache library: decode
 * attention, cache maintenance and causal prefill over the paged cache.
 *
 * The library implements the data-parallel hot path of PagedAttention as
 * the pages describe it:
 *   - "Efficient Memory Management for Large Language Model Serving with
 *     PagedAttention" (summary page, xasun.com article 3997), section 2:
 *     attention whose keys and values sit in non-contiguous, fixed-size
 *     physical blocks, fetched block by block through a per-sequence block
 *     table; a KV-cache manager maps logical to physical blocks and
 *     allocates them on demand; section 1: reference counts plus
 *     copy-on-write let parallel samples and shared prefixes share blocks.
 *   - "PyTorch-CUDA-v2.9 image enables PagedAttention" (jsqmd.com 164355),
 *     PagedAttention section and workflow list: pages of 16 tokens, a page
 *     table from logical position to physical page, a global page pool,
 *     each decode step appends the new token's key/value.
 *   - "GPT-OSS memory management: PagedAttention explained"
 *     (yongjin360.com 448593), section 2.2: the table tells where token N's
 *     key/value lives.
 *
 * Conventions for every call below
 *   Layout   caches are [num_blocks][num_kv_heads][block_size][head_size]
 *            (row-major, contiguous); token t of a sequence lives in block
 *            block_table[t / block_size] at offset t % block_size; query
 *            head h reads KV head h / (num_heads / num_kv_heads).  q and out
 *            are [num_seqs][num_heads][head_size], contiguous.
 *   Pointers "device" pointers must be CUDA device memory of the current
 *            device; every device buffer must start on a 16-byte boundary.
 *   Ownership the caller owns every buffer.  The library allocates no
 *            device memory and keeps no pointer after a call returns.  The
 *            block manager owns host memory only (create/destroy).
 *   Streams  GPU calls are asynchronous on the given cudaStream_t (passed as
 *            void*, NULL = the legacy default stream); they never
 *            synchronise, except pkv_read_device_errors.  The stream must
 *            belong to the current device (not checked: the call's kernels,
 *            scratch and error word are the current device's).
 *   Errors   argument errors are found on the host before anything is
 *            launched and return a status with nothing launched.  A failed
 *            launch returns PKV_ERR_CUDA.  Conditions only the device can see
 *            (a block id outside the pool, a slot outside the pool, a context
 *            longer than the table or than max_context_len) make the kernel
 *            skip the offending access and set a sticky bit, read with
 *            pkv_read_device_errors.  No kernel traps.
 *   Threads  calls are thread-safe as long as concurrent calls use
 *            different workspaces.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PKV_OK = 0,
    PKV_ERR_INVALID_ARG = 1,    /* null pointer, negative size, misaligned buffer ... */
    PKV_ERR_UNSUPPORTED = 2,    /* outside the supported domain (dtype, head_size, ...) */
    PKV_ERR_CUDA = 3,           /* a CUDA runtime call or a launch failed */
    PKV_ERR_OUT_OF_BLOCKS = 4,  /* block manager: not enough free blocks (state unchanged) */
    PKV_ERR_NOT_FOUND = 5,      /* block manager: unknown sequence id / id already in use */
    PKV_ERR_WORKSPACE = 6,      /* workspace missing or smaller than required */
    PKV_ERR_DEVICE_CHECK = 7    /* a device-side check fired (see PKV_DEVERR_*) */
} pkv_status;

typedef enum { PKV_F32 = 0, PKV_F16 = 1, PKV_BF16 = 2 } pkv_dtype;

/* Sticky device-side check bits. */
#define PKV_DEVERR_BLOCK_ID 1u  /* a block-table entry outside [0, num_blocks) */
#define PKV_DEVERR_SLOT 2u      /* a slot outside [0, num_blocks * block_size) */
#define PKV_DEVERR_CONTEXT 4u   /* context_len < 0, > max_blocks_per_seq * block_size or > max_context_len */
#define PKV_DEVERR_COPY_ID 8u   /* a copy_blocks pair outside [0, num_blocks) */
#define PKV_DEVERR_WAIT 16u     /* a bounded wait for an asynchronous copy gave up */
#define PKV_DEVERR_COPY_OVERLAP 32u /* copy pairs whose result would depend on their order */

const char* pkv_status_string(pkv_status status);
const char* pkv_version(void);

/* ---------------------------------------------------------------------------
 * paged_attention_decode -- one decode step of attention for a batch.
 *
 * Defines: out[s, h, :] = sum_t softmax_t(scale * q[s,h] . K_s[t]) V_s[t] over
 * t < context_lens[s], with K_s[t] = k_cache[block_tables[s][t / bs]][h / G]
 * [t % bs] (V likewise) -- the summary page of the SOSP 2023 paper, section 2
 * (attention over non-contiguous blocks through the block table) and
 * section 1 (exact: the output distribution is unchanged).  A sequence with
 * context_lens[s] == 0 gets an all-zero output.
 *
 *   out            device, [num_seqs][num_heads][head_size], dtype (written)
 *   q              device, [num_seqs][num_heads][head_size], dtype
 *   k_cache        device, [num_blocks][num_kv_heads][block_size][head_size], dtype
 *   v_cache        device, same shape as k_cache
 *   block_tables   device, int32 [num_seqs][max_blocks_per_seq]; entries past
 *                  ceil(context_len / block_size) are never read
 *   context_lens   device, int32 [num_seqs]; tokens to attend (includes the
 *                  step's own token once reshape_and_cache wrote it)
 *   scale          softmax scale (usually 1/sqrt(head_size))
 *   num_kv_heads   KV heads; num_heads must be a multiple (G = num_heads /
 *                  num_kv_heads, any value: MHA, GQA and MQA)
 *   block_size     tokens per block, 16 or 32
 *   num_seqs ... max_blocks_per_seq   the sizes above
 *   max_context_len host-known upper bound of context_lens; sizes the
 *                  workspace and picks the split.  0 means max_blocks_per_seq
 *                  * block_size (the workspace must then be sized for that)
 *   dtype          element type of q, caches and out (all the same)
 *   partition_size tokens per split-context partition: 0 = library choice
 *                  (a per-call size between 8 and 16 blocks; for G >= 4,
 *                  16 and 64, or 16 and 32 over an FP8 cache); otherwise a
 *                  multiple of block_size, at most 32 * block_size.
 *                  Contexts longer than one partition are
 *                  processed in parallel pieces whose softmax statistics a
 *                  second kernel merges (log-sum-exp reduction).
 *   workspace      device scratch of at least
 *                  paged_attention_workspace_size(...) bytes.  Its first 256
 *                  bytes hold scheduling counters that must be zero before
 *                  the first use (paged_attention_workspace_init, or a
 *                  zero-filled allocation); every call leaves them zero,
 *                  also one whose bounded waits gave up (PKV_DEVERR_WAIT).
 *                  Calls that run concurrently need separate workspaces.
 *   stream         cudaStream_t (void*), may be NULL
 *
 * Supported: dtype f32/f16/bf16, head_size 64 or 128, block_size 16 or 32,
 * any G, num_seqs <= 16384.  Anything else: PKV_ERR_UNSUPPORTED.  With f16
 * or bf16 elements, G >= 16 and partition_size 0, the call runs on the
 * tcgen05 tensor cores: the rows of each product are the group's query heads
 * (slices of up to 128), and the key tiles of all (sequence, KV head, slice)
 * units are split into ranges of equal cost over one CTA per SM, whose
 * partial results the merge kernel combines.  Otherwise groups of more than
 * 8 query heads are processed in slices of 8 heads that stream the same K/V
 * tiles at about the same time (the repeats come from L2).
 * ------------------------------------------------------------------------- */
pkv_status paged_attention_decode(void* out, const void* q, const void* k_cache,
                                  const void* v_cache, const int32_t* block_tables,
                                  const int32_t* context_lens, float scale, int num_kv_heads,
                                  int block_size, int num_seqs, int num_heads, int head_size,
                                  int num_blocks, int max_blocks_per_seq, int max_context_len,
                                  pkv_dtype dtype, int partition_size, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * paged_attention_decode_append -- reshape_and_cache of one new token per
 * sequence fused into paged_attention_decode (one launch fewer per step).
 *
 * Defines exactly what reshape_and_cache(key, value, ..., slot_mapping)
 * followed by paged_attention_decode(...) defines: the decode step appends
 * the new token's key/value ("PyTorch-CUDA-v2.9 image enables
 * PagedAttention", PagedAttention section) and attends over the context
 * including it.  Token s's rows key[s][g] / value[s][g] (token stride in
 * elements, multiple of 16 bytes) go to slot slot_mapping[s] (int64,
 * device); a negative slot means no new token for that sequence.  The slot
 * must be the slot of position context_lens[s] - 1 (the block-table entry of
 * that position and its offset); otherwise nothing is written for that
 * sequence and PKV_DEVERR_SLOT is set.  The block holding the slot must not
 * be shared with another sequence (copy_blocks first, as for
 * reshape_and_cache).  Every other argument, the workspace and the errors
 * are those of paged_attention_decode.
 * ------------------------------------------------------------------------- */
pkv_status paged_attention_decode_append(void* out, const void* q, const void* key,
                                         const void* value, void* k_cache, void* v_cache,
                                         const int64_t* slot_mapping, const int32_t* block_tables,
                                         const int32_t* context_lens, float scale,
                                         int num_kv_heads, int block_size, int num_seqs,
                                         int num_heads, int head_size, int num_blocks,
                                         int max_blocks_per_seq, int max_context_len,
                                         int64_t key_token_stride, int64_t value_token_stride,
                                         pkv_dtype dtype, int partition_size, void* workspace,
                                         size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * FP8 KV cache ("GPT-OSS memory management: PagedAttention explained",
 * section 3.2: kv_cache_dtype configures the cache element type).
 *
 * The caches hold FP8 E4M3 codes (1 byte per element: 1 sign, 4 exponent bits
 * with bias 7, 3 fraction bits, no infinities, 0x7f/0xff NaN, largest finite
 * 448), same layout [num_blocks][num_kv_heads][block_size][head_size], and a
 * cache element stands for code * scale with one scale for all of K
 * (k_scale) and one for all of V (v_scale), both > 0.
 *
 * paged_attention_decode_fp8kv: paged_attention_decode over such caches:
 *   out[s, h, :] = sum_t softmax_t(scale * q . (k_scale * K_s[t])) v_scale * V_s[t],
 * q and out in `dtype` (f32, f16 or bf16).  Workspace, partitioning, checks
 * and errors as for paged_attention_decode (the workspace size does not
 * depend on the cache type).  With 16-bit q the products run on the tensor
 * cores in fp16 (E4M3 is exact in fp16; bf16 q is rounded to fp16 there, so
 * |q| must stay below 65504).
 *
 * reshape_and_cache_fp8kv: reshape_and_cache into such caches: each element
 * x of key (value) becomes e4m3(x / k_scale) (resp. v_scale), the quotient
 * correctly rounded in fp32 and then rounded to nearest-even E4M3,
 * saturating to +-448 (NaN stays NaN).  key/value are in `dtype`.
 * ------------------------------------------------------------------------- */
pkv_status paged_attention_decode_fp8kv(void* out, const void* q, const void* k_cache,
                                        const void* v_cache, const int32_t* block_tables,
                                        const int32_t* context_lens, float scale, float k_scale,
                                        float v_scale, int num_kv_heads, int block_size,
                                        int num_seqs, int num_heads, int head_size, int num_blocks,
                                        int max_blocks_per_seq, int max_context_len,
                                        pkv_dtype dtype, int partition_size, void* workspace,
                                        size_t workspace_bytes, void* stream);

pkv_status reshape_and_cache_fp8kv(const void* key, const void* value, void* k_cache,
                                  void* v_cache, const int64_t* slot_mapping, int num_tokens,
                                  int num_kv_heads, int head_size, int block_size, int num_blocks,
                                  int64_t key_token_stride, int64_t value_token_stride,
                                  pkv_dtype dtype, float k_scale, float v_scale, void* stream);

/* Bytes of workspace paged_attention_decode needs for these sizes (0 on bad
 * arguments).  partition_size as in paged_attention_decode. */
size_t paged_attention_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                      int head_size, int block_size, int max_context_len,
                                      pkv_dtype dtype, int partition_size);

/* The smallest partition size paged_attention_decode may use for these
 * arguments: the requested size, or for partition_size 0 the lower end of
 * the library's range (the kernel then picks, per call, a block multiple
 * between this and twice this that keeps the last round of work items full).
 * Contexts up to this length are never split.  0 on bad arguments. */
int paged_attention_partition_size(int num_heads, int num_kv_heads, int block_size,
                                   int max_context_len, int partition_size);

/* Zero the scheduling counters of a workspace (asynchronous memset). */
pkv_status paged_attention_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * reshape_and_cache -- write each new token's key and value into its slot.
 *
 * Defines: for every token i with slot = slot_mapping[i] >= 0 and every KV
 * head g: k_cache[slot / bs][g][slot % bs][:] = key[i][g][:] and likewise
 * for value; a negative slot means "skip".  A bit copy, no conversion.  The
 * decode step appends the new token's key/value ("PyTorch-CUDA-v2.9 image
 * enables PagedAttention", PagedAttention section; workflow list: prefill
 * writes the input tokens' KV into pages).
 *
 *   key, value     device, token i's head g at element i * *_token_stride +
 *                  g * head_size (strides in elements, multiples of
 *                  16 bytes / element size)
 *   k_cache, v_cache device caches (layout above)
 *   slot_mapping   device, int64 [num_tokens]
 *   num_blocks     pool size (slots >= num_blocks * block_size are skipped
 *                  and flag PKV_DEVERR_SLOT)
 * ------------------------------------------------------------------------- */
pkv_status reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                             const int64_t* slot_mapping, int num_tokens, int num_kv_heads,
                             int head_size, int block_size, int num_blocks,
                             int64_t key_token_stride, int64_t value_token_stride,
                             pkv_dtype dtype, void* stream);

/* ---------------------------------------------------------------------------
 * copy_blocks -- the copy-on-write block copy.
 *
 * Defines: for every layer l and pair i, block block_mapping[i][1] of
 * k_caches[l] and v_caches[l] becomes a copy of block block_mapping[i][0]
 * (summary page of the SOSP 2023 paper, sections 1 and 2: copy-on-write
 * when parallel samples or shared prefixes diverge).  A bit copy of
 * block_bytes bytes per block.  Pairs are copied in parallel, so the result
 * is that of copying them in any order only if destinations are distinct and
 * no destination is also a source: a pair that shares its destination with
 * another pair, or whose destination or source is another pair's source or
 * destination, is skipped and sets PKV_DEVERR_COPY_OVERLAP (the other pairs
 * are copied).  Several pairs may share one source (one shared block copied
 * for several writers).  Each CTA checks its pair against the whole mapping,
 * which adds num_pairs * 16 bytes of (cached) reads per block copied.
 *
 *   k_caches, v_caches HOST arrays of num_layers device pointers
 *   block_mapping  device, int64 [num_pairs][2] = (src, dst)
 *   num_blocks     pool size of every cache (ids outside flag
 *                  PKV_DEVERR_COPY_ID and are skipped)
 *   block_bytes    bytes of one block of one cache (num_kv_heads *
 *                  block_size * head_size * element size), a multiple of 16
 *   num_layers     1 .. 256
 * ------------------------------------------------------------------------- */
pkv_status copy_blocks(void* const* k_caches, void* const* v_caches, int num_layers,
                       const int64_t* block_mapping, int num_pairs, int num_blocks,
                       int64_t block_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * paged_attention_decode_noalloc -- paged_attention_decode without a
 * workspace argument.  The pages have no counterpart: this entry point only
 * serves callers that cannot allocate device memory, such as a plug-in
 * inside a host framework that owns every device allocation through its own
 * arena, or a latency-critical loop that cannot accept cudaMalloc's implicit
 * device synchronisation.  The caller still passes the inputs and the output.
 *
 * Scratch: one fixed array of PKV_NOALLOC_SCRATCH_BYTES (16 MiB) inside the
 * library, reserved on every GPU that loads the library until the process
 * exits.  Sizes whose workspace (paged_attention_workspace_size) exceeds it
 * are rejected with PKV_ERR_WORKSPACE and nothing is launched; all other
 * argument checks and results are those of paged_attention_decode.  The
 * call allocates nothing (no cudaMalloc, no cudaFree): it clears the
 * scheduling counters at the head of the array with an asynchronous memset
 * on the stream, then launches.
 *
 * Set-up: the first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  The stream must belong to the current device,
 * whose array the call uses (not checked).
 *
 * Sharing: every call, on every stream and thread, uses the same array, which
 * keeps the previous call's contents.  Calls that overlap on the GPU race on
 * it; serialise them (one stream, or events between streams).
 * ------------------------------------------------------------------------- */
#define PKV_NOALLOC_SCRATCH_BYTES (16u << 20)

pkv_status paged_attention_decode_noalloc(void* out, const void* q, const void* k_cache,
                                          const void* v_cache, const int32_t* block_tables,
                                          const int32_t* context_lens, float scale,
                                          int num_kv_heads, int block_size, int num_seqs,
                                          int num_heads, int head_size, int num_blocks,
                                          int max_blocks_per_seq, int max_context_len,
                                          pkv_dtype dtype, int partition_size, void* stream);

/* ---------------------------------------------------------------------------
 * swap_blocks -- block copy between two pools, typically the GPU pool and a
 * pinned host pool ("Efficient Memory Management for Large Language Model
 * Serving with PagedAttention" summary page, section 2: the KV-cache manager
 * keeps a block pool in GPU memory and one in CPU memory for swapping; the
 * scheduler recovers preempted requests by swapping).
 *
 * Defines: for every cache c < num_caches and pair i, block
 * block_mapping[i][1] of dst_caches[c] becomes a bit copy of block
 * block_mapping[i][0] of src_caches[c] (block_bytes bytes each).
 *   src_caches, dst_caches  HOST arrays of num_caches pointers (e.g. the K
 *                  and V caches of every layer, <= 512); each pointer is
 *                  device memory or pinned (page-locked, mapped) host memory,
 *                  checked on the host (PKV_ERR_INVALID_ARG otherwise)
 *   block_mapping  int64 [num_pairs][2] (src, dst) in device or pinned host
 *                  memory; ids outside [0, src_num_blocks) / [0,
 *                  dst_num_blocks) are skipped and flag PKV_DEVERR_COPY_ID
 * Destinations must be distinct: pairs that share a destination are skipped
 * and set PKV_DEVERR_COPY_OVERLAP.  Asynchronous on the stream; the host pool
 * must stay alive until the stream has passed the copy.
 * ------------------------------------------------------------------------- */
pkv_status swap_blocks(const void* const* src_caches, void* const* dst_caches, int num_caches,
                       const int64_t* block_mapping, int num_pairs, int src_num_blocks,
                       int dst_num_blocks, int64_t block_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * paged_attention_prefill -- causal attention of a batch of prompts, or of
 * prompt chunks, whose keys and values are already in the paged cache.
 *
 * Defines: sequence s has L = context_lens[s] tokens in its blocks and n =
 * query_start_loc[s+1] - query_start_loc[s] queries, the last n of those
 * tokens.  For query i (row query_start_loc[s] + i of q) at position
 * p = L - n + i,
 *   out[row, h, :] = sum_{t <= p} softmax_t(scale * q[row,h] . K_s[t]) V_s[t]
 * with K_s / V_s read through the block table as in the decode call.  The
 * pages' serving workflow ("PyTorch-CUDA-v2.9 image enables PagedAttention",
 * workflow list, and its chunked-prefill usage notes): the prompt's keys and
 * values are first written into pages (reshape_and_cache), then attended
 * causally; a chunk of a long prompt attends to every earlier chunk's keys
 * already in the pages plus its own.  n == L is a whole prompt; n == 1 is a
 * decode step.
 *
 *   out            device, [num_tokens][num_heads][head_size], dtype (written;
 *                  rows of every sequence's queries)
 *   q              device, [num_tokens][num_heads][head_size], dtype
 *   k_cache, v_cache, block_tables   as in paged_attention_decode
 *   context_lens   device, int32 [num_seqs]: tokens in the cache for s,
 *                  including this call's queries (written beforehand)
 *   query_start_loc device, int32 [num_seqs + 1], non-decreasing,
 *                  query_start_loc[0] = 0, query_start_loc[num_seqs] = num_tokens
 *   scale          softmax scale, finite and > 0 (else PKV_ERR_INVALID_ARG)
 *   max_query_len  host-known bound of n over the batch (> 0 unless
 *                  num_tokens == 0); sizes the grid
 *   dtype          f16 or bf16 (q, caches and out the same); the products
 *                  run on the tensor cores with fp32 accumulation and the
 *                  softmax weights rounded to dtype before the product with V
 *
 * The kernel is persistent (one CTA per SM) and takes its work items from a
 * counter the library owns: each call takes the next of 64 counters of the
 * device, and its last CTA leaves it at zero, on every path.  At most 64
 * prefill calls may run at the same time on one device (streams running in
 * parallel); calls on one stream run one after another.
 *
 * Device checks: n < 0, n > L, n > max_query_len, L > max_blocks_per_seq *
 * block_size or queries outside [0, num_tokens) set PKV_DEVERR_CONTEXT and
 * the sequence's rows are not written; a block id outside the pool sets
 * PKV_DEVERR_BLOCK_ID and reads as zeros.
 * Supported: head_size 64 or 128, block_size 16 or 32, G = num_heads /
 * num_kv_heads from 1 to 128 (a query tile of 128 rows holds floor(128 / G)
 * queries of G heads), num_blocks * num_kv_heads * block_size < 2^31.
 * f32: PKV_ERR_UNSUPPORTED.
 * ------------------------------------------------------------------------- */
pkv_status paged_attention_prefill(void* out, const void* q, const void* k_cache,
                                   const void* v_cache, const int32_t* block_tables,
                                   const int32_t* context_lens, const int32_t* query_start_loc,
                                   float scale, int num_tokens, int num_seqs, int num_heads,
                                   int num_kv_heads, int head_size, int block_size,
                                   int num_blocks, int max_blocks_per_seq, int max_query_len,
                                   pkv_dtype dtype, void* stream);

/* Synchronise the stream, return the sticky device-check bits of the
 * current device in *bits and clear them.  Returns PKV_ERR_DEVICE_CHECK if
 * any bit was set, else PKV_OK (or PKV_ERR_CUDA). */
pkv_status pkv_read_device_errors(void* stream, uint32_t* bits);

/* For tests of the failure path: every wait of the decode and prefill kernels
 * for an asynchronous copy, a tensor-core commit or another warp's result
 * gives up after `polls` polls (each may suspend the thread for a short
 * hardware-defined time), skips the rest of its work, lets the copies it
 * already issued land, frees what it holds and sets PKV_DEVERR_WAIT; the
 * outputs of that call are then undefined.  polls = 0 gives up at the first
 * wait; polls < 0 restores the default (2^22, far beyond any real latency).
 * Process-wide; applies to calls launched after it returns.  polls above
 * 2^32 - 1: PKV_ERR_INVALID_ARG. */
pkv_status pkv_set_wait_limit(int64_t polls);

/* ---------------------------------------------------------------------------
 * Host block manager (KV-cache manager of the summary page, section 2; the
 * global page pool of the PyTorch-CUDA page's workflow list).  Host memory
 * only; not thread-safe (one manager per thread or external locking).
 *
 * Policy: free blocks are handed out first-in first-out from a list whose
 * initial order is free_order (NULL = 0..num_blocks-1); freed blocks go to
 * the tail.  Allocation is all-or-nothing: when too few blocks are free the
 * call returns PKV_ERR_OUT_OF_BLOCKS and changes nothing (the summary page,
 * section 2: all-or-nothing eviction).  Appending into a shared, partially
 * filled last block first moves the sequence to a fresh copy and reports
 * the (src, dst) pair, which the caller passes to copy_blocks before
 * reshape_and_cache writes the token.
 * ------------------------------------------------------------------------- */
typedef struct pkv_block_manager pkv_block_manager;

pkv_status pkv_bm_create(int num_blocks, int block_size, const int32_t* free_order,
                         pkv_block_manager** out);
void pkv_bm_destroy(pkv_block_manager* bm);
/* New sequence holding num_tokens tokens (ceil(num_tokens / block_size) blocks). */
pkv_status pkv_bm_allocate(pkv_block_manager* bm, int64_t seq_id, int num_tokens);
/* child shares all of parent's blocks (each reference count + 1). */
pkv_status pkv_bm_fork(pkv_block_manager* bm, int64_t parent, int64_t child);
/* Slot of the sequence's next token; cow_src and cow_dst receive the copy to make
 * first, or -1/-1. */
pkv_status pkv_bm_append_slot(pkv_block_manager* bm, int64_t seq_id, int64_t* slot,
                              int32_t* cow_src, int32_t* cow_dst);
/* append_slot for n sequences in order: slots[n]; cow_pairs[2 * k] for the
 * k-th copy, *num_cow copies.  Stops at the first failure and returns its
 * status; *num_done tells how many sequences were served. */
pkv_status pkv_bm_append_slots(pkv_block_manager* bm, const int64_t* seq_ids, int n,
                               int64_t* slots, int64_t* cow_pairs, int* num_cow, int* num_done);
/* Swap a whole sequence from manager bm to manager host (e.g. GPU pool to
 * host pool; the reverse call swaps it back in), all or nothing: host gets
 * the sequence with fresh private blocks (sharing ends at a swap), bm drops
 * its references.  pairs[2 * j], pairs[2 * j + 1] = (block in bm, block in
 * host) for the j-th logical block, the copies to pass to swap_blocks;
 * *num_pairs = the sequence's block count.  PKV_ERR_OUT_OF_BLOCKS (nothing
 * changed) if host has too few free blocks; PKV_ERR_INVALID_ARG if capacity
 * is too small or the block sizes differ. */
pkv_status pkv_bm_swap_out(pkv_block_manager* bm, pkv_block_manager* host, int64_t seq_id,
                           int64_t* pairs, int capacity, int* num_pairs);
pkv_status pkv_bm_free(pkv_block_manager* bm, int64_t seq_id);
/* Copy the sequence's table into out[0 .. capacity); *num_blocks = its length. */
pkv_status pkv_bm_block_table(const pkv_block_manager* bm, int64_t seq_id, int32_t* out,
                              int capacity, int* num_blocks);
/* Tables and lengths of n sequences: tables[n][max_blocks_per_seq] (unused
 * entries -1), context_lens[n]. */
pkv_status pkv_bm_fill_tables(const pkv_block_manager* bm, const int64_t* seq_ids, int n,
                              int32_t* tables, int max_blocks_per_seq, int32_t* context_lens);
int pkv_bm_num_free(const pkv_block_manager* bm);
int pkv_bm_seq_len(const pkv_block_manager* bm, int64_t seq_id);   /* -1 if unknown */
int pkv_bm_ref_count(const pkv_block_manager* bm, int32_t block);  /* -1 if out of range */
/* Written token slots / slots of all blocks in use (0 if none in use). */
double pkv_bm_utilisation(const pkv_block_manager* bm);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
