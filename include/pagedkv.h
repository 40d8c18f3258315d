/*
 * pagedkv.h -- C ABI of the paged KV cache decode library (libpagedkv.so).
 *
 * One decode step of a transformer layer over a paged KV cache:
 *
 *   kv_cache_append         scatter each new token's K and V rows into its slot
 *   paged_attention_decode  out = softmax(scale * q K^T) V per query head,
 *                           reading K/V through per-sequence block tables
 *   paged_attention_decode_append   the two above in one launch
 *   paged_attention_decode_layers   the same over several layers of one step
 *                           in one launch
 *   paged_attention_prefill chunked prefill: a chunk of query tokens per
 *                           sequence, causal over the same cache
 *   kv_cache_copy_blocks, kv_cache_gather_blocks, kv_cache_scatter_blocks
 *                           whole-block moves over every layer's caches
 *                           (copy-on-write, swap-out, swap-in)
 *   kv_pool_*               host bookkeeping of physical blocks: allocate,
 *                           free, reference counts for shared prefixes, fork,
 *                           per-step slots (with copy-on-write)
 *
 * Sources for what is computed:
 *   - "Module 23: Serving", section 23.4 (Paged Attention): the cache lives in
 *     fixed-size blocks of 16 tokens, allocated as a sequence grows, with a
 *     per-sequence table mapping positions to blocks; sequences that share a
 *     prefix can share its blocks.
 *   - "Designing an LLM serving system", section "Paged attention": a page
 *     table per sequence; logical positions map to physical blocks through an
 *     indirection; shared blocks for a common prompt.
 *   - "Scaling LLM serving", section "The KV cache" (Share key/value heads):
 *     grouped-query attention, each key/value head shared by a group of query
 *     heads. Groups are contiguous: query head h reads kv head h / (Hq / Hkv).
 *   - "Module 23: Serving", section 23.2 (Prefill and Decode): a decode step
 *     reads the whole KV cache for one new token per sequence.
 *
 * Conventions for every call:
 *   - Device pointers are CUDA global-memory addresses on the current device.
 *     The caller owns every buffer, the workspace included. The library never
 *     allocates or frees device memory and never synchronises, except where a
 *     call says so (paged_attention_read_status).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Work is
 *     enqueued on it; kernels are launched with programmatic dependent launch,
 *     so consecutive calls on one stream may overlap their prologues. All calls
 *     that launch work can be captured into a CUDA graph.
 *   - Return value: KV_OK (0) or a negative kv_status. Argument checks happen on
 *     the host before anything is enqueued; on KV_ERR_ARG nothing is launched.
 *     KV_ERR_CUDA means a launch failed (cudaGetLastError was not cudaSuccess).
 *   - Element type: dtype is KV_DTYPE_BF16 or KV_DTYPE_FP16 (2 bytes per
 *     number either way: "Module 23: Serving", section 23.1, equation
 *     Memory_KV), the same for q, out, the caches and the new tokens of a call.
 *     Arithmetic is fp32 whatever the element type. Head dimension D must be 64
 *     or 128. Block size is fixed at KV_BLOCK_TOKENS = 16 tokens.
 *
 * Layouts (row-major; "elem" = bf16 or fp16 as dtype says):
 *   k_cache, v_cache   [num_blocks][16][Hkv][D]  elem, one tensor each for K, V
 *   q, out             [B][Hq][D]               elem
 *   k_new, v_new       [T][Hkv][D]              elem
 *   slot_mapping       [T]                      int64; slot = block*16 + offset,
 *                                                negative = padding (skipped)
 *   block_tables       [B][W]                   int32 physical block ids; row b
 *                                                holds ceil(context_lens[b]/16)
 *                                                valid entries, the rest unread
 *   context_lens       [B]                      int32 tokens cached for sequence
 *                                                b, this step's token included
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define KV_API __attribute__((visibility("default")))
#else
#define KV_API
#endif

typedef int kv_status;

#define KV_OK 0
#define KV_ERR_ARG (-1)    /* bad argument; nothing was done                       */
#define KV_ERR_OOM (-2)    /* block pool has too few free blocks; nothing changed  */
#define KV_ERR_STATE (-3)  /* pool state forbids it (free of a free block, ...)    */
#define KV_ERR_CUDA (-4)   /* a CUDA runtime call failed                           */

#define KV_DTYPE_BF16 0
#define KV_DTYPE_FP16 1
#define KV_BLOCK_TOKENS 16

/* Bits of the device status word kept in the attention workspace. */
#define KV_STATUS_BAD_BLOCK_ID 1   /* a table entry was outside [0, num_blocks)   */
#define KV_STATUS_BAD_CONTEXT 2    /* a context length was < 0 or > 16 * W        */
#define KV_STATUS_WAIT_TIMEOUT 4   /* an internal pipeline wait gave up (~1 s)    */
#define KV_STATUS_BAD_SLOT 8       /* an append slot was >= num_blocks * 16       */

typedef struct CUstream_st *kv_stream_t; /* same type as cudaStream_t */

/* ------------------------------------------------------------------------ */
/* Append ("Module 23: Serving", 23.4: blocks are filled as a sequence grows) */
/* ------------------------------------------------------------------------ */
/*
 * For every i in [0, T) with slot_mapping[i] >= 0:
 *   k_cache[slot/16][slot%16][:][:] = k_new[i][:][:]   (all Hkv heads, bitwise)
 *   v_cache[slot/16][slot%16][:][:] = v_new[i][:][:]
 * Every other cache byte is left unchanged. Non-negative slots must be
 * distinct (two tokens writing one slot race). A slot >= num_blocks*16 is not
 * written; if error_flag is non-NULL (a device int32), KV_STATUS_BAD_SLOT is
 * OR-ed into it. All pointers are device pointers, 16-byte aligned.
 * T = 0 is a no-op.
 */
KV_API kv_status kv_cache_append(const void *k_new, const void *v_new,
                          void *k_cache, void *v_cache,
                          const int64_t *slot_mapping, int T,
                          int num_blocks, int Hkv, int D, int dtype,
                          int32_t *error_flag, kv_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Decode attention ("Module 23: Serving", 23.2 and 23.4; "Scaling LLM       */
/* serving", "The KV cache")                                                 */
/* ------------------------------------------------------------------------ */
/*
 * Bytes of device workspace paged_attention_decode needs for these sizes on
 * the current device (it depends on the device's SM count). Returns 0 for
 * invalid sizes, or when no CUDA device can be queried. The workspace holds a status word, split-K partial results
 * and one counter per (sequence, kv head) work item.
 */
KV_API size_t paged_attention_workspace_size(int B, int Hq, int Hkv, int D);

/*
 * Zero a workspace (cudaMemsetAsync on `stream`). A workspace must be zeroed
 * once before its first use, and again after a call reported
 * KV_STATUS_WAIT_TIMEOUT; between calls it stays valid by itself.
 */
KV_API kv_status paged_attention_workspace_init(void *workspace, size_t workspace_bytes,
                                         kv_stream_t stream);

/*
 * For each sequence b with c = context_lens[b], each query head h in [0, Hq)
 * and j = h / (Hq / Hkv):
 *   K_t = k_cache[block_tables[b][t/16]][t%16][j][:],  V_t likewise, t < c
 *   out[b][h][:] = sum_t softmax_t(scale * <q[b][h], K_t>) V_t
 * computed with fp32 arithmetic (16-bit inputs and output of the element
 * type). c = 0 gives out[b][h][:] = 0. The result does not depend on which
 * physical blocks hold the tokens, only on the logical order, and is bitwise
 * reproducible.
 *
 * q, out, k_cache, v_cache, block_tables, context_lens, workspace: device
 * pointers (the first four 16-byte aligned, workspace 256-byte aligned).
 * workspace_bytes must be >= paged_attention_workspace_size(B, Hq, Hkv, D).
 * Requirements: B >= 0, W >= 1, num_blocks >= 1, Hq % Hkv == 0, D in {64, 128}.
 * Bad table entries or context lengths are not checked on the host (the data
 * is on the device): the kernel never reads outside the cache or the table
 * row, and records KV_STATUS_BAD_BLOCK_ID / KV_STATUS_BAD_CONTEXT in the
 * workspace status word (see paged_attention_read_status); the output of an
 * affected sequence is then unspecified.
 * Concurrent calls must not share a workspace.
 */
KV_API kv_status paged_attention_decode(void *out, const void *q,
                                 const void *k_cache, const void *v_cache,
                                 const int32_t *block_tables, int max_blocks_per_seq,
                                 const int32_t *context_lens, int B,
                                 int num_blocks, int Hq, int Hkv, int D,
                                 float scale, int dtype,
                                 void *workspace, size_t workspace_bytes,
                                 kv_stream_t stream);

/*
 * Copy the workspace status word to *status_out (host int32), synchronising
 * `stream` first; if clear != 0, reset it to 0 afterwards. 0 = no error seen.
 */
KV_API kv_status paged_attention_read_status(const void *workspace, int32_t *status_out,
                                      int clear, kv_stream_t stream);

/*
 * Append fused into decode: the same result as kv_cache_append(k_new, v_new,
 * k_cache, v_cache, slot_mapping, T = B, ...) followed by
 * paged_attention_decode(...), in one kernel launch. k_new/v_new are
 * [B][Hkv][D] elem (16-byte aligned), slot_mapping [B] int64 (device).
 * Sequence b's new token must be its last cached token: slot_mapping[b] ==
 * block_tables[b][(c-1)/16] * 16 + (c-1) % 16 with c = context_lens[b], and
 * its block must not be read by any other sequence of the batch (true for
 * blocks from kv_pool_append_slots). A negative slot appends nothing; any
 * other slot is not written, KV_STATUS_BAD_SLOT is recorded in the workspace
 * status word and that sequence's output is unspecified. ("Module 23:
 * Serving", section 23.4: a block fills as its sequence grows.)
 */
KV_API kv_status paged_attention_decode_append(void *out, const void *q,
                                               const void *k_new, const void *v_new,
                                               void *k_cache, void *v_cache,
                                               const int64_t *slot_mapping,
                                               const int32_t *block_tables, int max_blocks_per_seq,
                                               const int32_t *context_lens, int B,
                                               int num_blocks, int Hq, int Hkv, int D,
                                               float scale, int dtype,
                                               void *workspace, size_t workspace_bytes,
                                               kv_stream_t stream);

/*
 * Several layers of one decode step in one launch ("Module 23: Serving",
 * section 23.1, equation Memory_KV: every layer keeps its own K and V for every
 * token, so a step reads num_layers caches through the same block tables).
 * For l in [0, num_layers) it gives the result of
 *   paged_attention_decode_append(out + l*B*Hq*D, q + l*B*Hq*D,
 *       k_new + l*B*Hkv*D, v_new + l*B*Hkv*D,
 *       k_cache + l*cache_layer_stride, v_cache + l*cache_layer_stride, ...)
 * (or of paged_attention_decode when k_new, v_new and slot_mapping are all
 * NULL), with the same block_tables, context_lens and slot_mapping for every
 * layer. Offsets are in elements: q and out are [num_layers][B][Hq][D], k_new
 * and v_new [num_layers][B][Hkv][D], all contiguous; layer l's caches start
 * cache_layer_stride elements after layer l-1's (a stacked
 * [num_layers][num_blocks][16][Hkv][D] pool has cache_layer_stride =
 * num_blocks*16*Hkv*D; any larger multiple of 8 up to 2^38 is accepted, the
 * same for K and V). The work of all layers is divided between the CTAs as one
 * sequence, so no layer waits for the previous one's split-K merges: a step
 * whose queries are all available at once (attention of every layer from the
 * same inputs, as a benchmark step is) pays the per-launch start-up and tail
 * once. In a transformer forward, layer l+1's q is computed from layer l's
 * output, so such a caller launches per layer instead.
 * workspace_bytes >= paged_attention_workspace_size_layers(B, Hq, Hkv, D,
 * num_layers); the other requirements, checks and the status word are those of
 * paged_attention_decode_append (a bad slot is reported once, not per layer).
 * num_layers >= 1; num_layers = 1 equals the single-layer calls.
 */
KV_API size_t paged_attention_workspace_size_layers(int B, int Hq, int Hkv, int D, int num_layers);
KV_API kv_status paged_attention_decode_layers(void *out, const void *q,
                                               const void *k_new, const void *v_new,
                                               void *k_cache, void *v_cache,
                                               size_t cache_layer_stride, int num_layers,
                                               const int64_t *slot_mapping,
                                               const int32_t *block_tables, int max_blocks_per_seq,
                                               const int32_t *context_lens, int B,
                                               int num_blocks, int Hq, int Hkv, int D,
                                               float scale, int dtype,
                                               void *workspace, size_t workspace_bytes,
                                               kv_stream_t stream);

/*
 * The same decode as paged_attention_decode, for callers that cannot allocate
 * device memory (for example a plugin inside a host program that owns every
 * device allocation, or code that must not trigger cudaMalloc's implicit
 * device synchronisation). The pages have no counterpart: it changes where
 * the split-K scratch lives, not what is computed.
 *
 * The scratch is one fixed array of KV_NOALLOC_SCRATCH_BYTES (16 MiB) inside
 * the library, present on every GPU that loads it until the process exits.
 * The caller still passes inputs and outputs; nothing is allocated or freed.
 * Sizes whose scratch (paged_attention_workspace_size) exceeds the array are
 * rejected with KV_ERR_ARG. The first call on a device looks up the array's
 * device address (cudaGetSymbolAddress, with that device current); make that
 * first call before any stream capture. The address is looked up again when
 * the device's current context has changed since; it cannot tell a context
 * that cudaDeviceReset destroyed from a new one at the same handle, so do not
 * call it across a cudaDeviceReset. Every check runs before anything is
 * enqueued; a call that goes ahead clears the array's status word and counters
 * on `stream`, then launches the kernel. All calls share the one array: calls
 * that can overlap on the GPU (other streams, other threads) race and give
 * wrong results; serialise them. Device data errors are guarded as in
 * paged_attention_decode but cannot be read back here.
 */
#define KV_NOALLOC_SCRATCH_BYTES (16u << 20)
KV_API kv_status paged_attention_decode_noalloc(void *out, const void *q,
                                                const void *k_cache, const void *v_cache,
                                                const int32_t *block_tables, int max_blocks_per_seq,
                                                const int32_t *context_lens, int B,
                                                int num_blocks, int Hq, int Hkv, int D,
                                                float scale, int dtype, kv_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Chunked prefill over the paged cache                                      */
/* ------------------------------------------------------------------------ */
/*
 * For each sequence b, the n_b = query_start[b+1] - query_start[b] rows
 * q[query_start[b] ..] are the queries of the last n_b tokens of its context
 * (context_lens[b] = c_b tokens, this chunk included: append its K/V first with
 * kv_cache_append). Chunk token i sits at position p = c_b - n_b + i and
 * attends causally to positions 0..p:
 *   out[query_start[b] + i][h] = sum_{t <= p} softmax_t(scale * <q[.][h], K_t>) V_t
 * with kv head h / (Hq / Hkv) and K_t, V_t read through block_tables as for the
 * decode. ("Module 23: Serving", section 23.2, Prefill and Decode; "Designing an
 * LLM serving system", section "Scheduling: when prefill meets decode":
 * chunked prefill.) n_b = c_b is a whole prompt; n_b = 1 is a decode step.
 *
 * q, out: [T][Hq][D] device, T = query_start[B]; query_start: [B+1] device
 * int32, non-decreasing from 0; max_query_len >= every n_b (it sizes the
 * grid). Tensor cores (tcgen05.mma with tensor-memory accumulators; mma.sync
 * with KV_OPT_PREFILL_PATH = 2), fp32 accumulation, the probabilities rounded
 * to the element type before they multiply V. No workspace. The default
 * kernel takes 256 query rows of one (sequence, kv head) per CTA, so
 * ceil(max_query_len * Hq / Hkv / 256) must be <= 65535. Data errors are
 * OR-ed into *error_flag (device int32, may be NULL): KV_STATUS_BAD_CONTEXT
 * when n_b > c_b, c_b > 16 * max_blocks_per_seq or n_b > max_query_len (that
 * sequence's rows are not written), KV_STATUS_BAD_BLOCK_ID for ids outside the
 * pool (block 0 is read instead), KV_STATUS_WAIT_TIMEOUT if an internal wait
 * gave up (~1 s; the output is not valid). B <= 65535, Hkv <= 65535, scale > 0.
 * Launched with programmatic dependent launch: query_start and context_lens
 * are read before the previous kernel in the stream has completed (it must not
 * write them); q, the caches, block_tables, out and *error_flag after.
 */
KV_API kv_status paged_attention_prefill(void *out, const void *q, const void *k_cache,
                                         const void *v_cache, const int32_t *block_tables,
                                         int max_blocks_per_seq, const int32_t *context_lens,
                                         const int32_t *query_start, int B, int max_query_len,
                                         int num_blocks, int Hq, int Hkv, int D, float scale,
                                         int dtype, int32_t *error_flag, kv_stream_t stream);

/*
 * Process-wide tuning switches (defaults are the tuned choices).
 *   KV_OPT_COMPUTE:   0 auto, 1 tensor cores (mma.sync, 16-bit inputs), 2 CUDA cores
 *   KV_OPT_COMBINE:   0 split-K merge fused into the last CTA of each work
 *                     item, 1 separate combine kernel
 *   KV_OPT_GRID:      0 auto (CTAs resident on all SMs), n > 0 launch n CTAs
 *                     (n is capped by what the workspace was sized for)
 *   KV_OPT_MIN_CHUNK: 0 auto, n > 0 minimum work positions per CTA
 *   KV_OPT_PRODUCER_LANES: 0 auto (2, or 4 with one kv head per unit),
 *                     1/2/4/8 lanes of the producer warp that issue tile
 *                     loads. The ring's stage count is rounded down to a
 *                     multiple of the lanes; a value that leaves fewer stages
 *                     than lanes (8 with D = 128) makes the decode calls
 *                     return KV_ERR_ARG.
 *   KV_OPT_HEAD_GROUP: 0 auto (4 if it divides Hkv, else 2 or 1), or 1/2/4 kv
 *                     heads per work unit when it divides Hkv. It changes
 *                     paged_attention_workspace_size: set it before sizing.
 *   KV_OPT_ITEM_COST: how the work is divided between CTAs. Every work unit
 *                     (one KV block of one kv-head group) is one work
 *                     position and every work item (a sequence's kv-head
 *                     group and query-head chunk) adds this many more for its
 *                     fixed cost; CTAs take equal ranges of positions.
 *                     0 auto, -1 none, 1..64 that many.
 *   KV_OPT_PREFILL_PATH: paged_attention_prefill on 0 auto (3), 1
 *                     tcgen05.mma with tensor-memory accumulators, one tile of
 *                     128 query rows per CTA (two CTAs per SM), 2 mma.sync,
 *                     3 tcgen05.mma, two tiles of 128 query rows per CTA
 *                     sharing each 128-token K/V tile (one CTA per SM).
 *   KV_OPT_TEST_DROP_LOAD: test hook for the timeout path, 0 (default) off;
 *                     n > 0: in the decode kernels' CTA that holds the
 *                     launch's first work unit, the tile load of its work
 *                     unit n - 1 is never issued, so the wait for it runs
 *                     out (after about a second): the call completes with
 *                     KV_STATUS_WAIT_TIMEOUT in the status word and its output
 *                     is not valid; the context stays usable (re-initialise
 *                     the workspace, as after any timed-out call).
 *   KV_OPT_TEST_SLOW_SOFTMAX: test hook for the hand-offs of the tcgen05
 *                     prefill kernels, 0 (default) off; 1: in every CTA the first
 *                     softmax warp waits about 30 microseconds before it hands
 *                     over P of the first tile, so the other warps run a tile
 *                     ahead of it. The output must not change.
 *   KV_OPT_OUT_F32:   debug switch for checking the arithmetic, 0 (default)
 *                     off; 1: `out` of the decode calls and of
 *                     paged_attention_prefill holds fp32 numbers (4 bytes
 *                     each, same shape, 16-byte aligned), the normalised
 *                     result before any rounding to the element type. The
 *                     other arguments keep their element type.
 *   KV_OPT_L2_POLICY: L2 priority of the decode kernels' K/V tile loads: 0
 *                     auto (evict normal for a multi-layer launch at D = 128,
 *                     evict first otherwise: the faster on every workload
 *                     measured), 1 evict first, 2 evict normal, 3 evict last.
 *   KV_OPT_EARLY_LOADS: 0 (default) off; 1: the caller promises that, for
 *                     every decode call in a stream, the kernel launched just
 *                     before it in that stream does not write the caches the
 *                     call reads (true for one launch per layer after a
 *                     projection kernel; false right after kv_cache_append
 *                     into the same cache, or after a previous step's launch
 *                     over the same caches). The decode kernels then issue
 *                     their first ring of K/V tile loads before that kernel
 *                     has finished (programmatic dependent launch); q, the
 *                     new rows, out and the workspace still wait for it. With
 *                     the promise broken, results are unspecified.
 * Kernels are launched with programmatic dependent launch. q, k_new, v_new,
 * the caches (unless KV_OPT_EARLY_LOADS is set), the workspace and out are
 * touched only after the previous kernel in the stream has completed;
 * block_tables and context_lens are read before that, so the kernel launched
 * just before a decode call must not write them.
 * Returns KV_ERR_ARG for an unknown key or value.
 */
#define KV_OPT_COMPUTE 1
#define KV_OPT_COMBINE 2
#define KV_OPT_GRID 3
#define KV_OPT_MIN_CHUNK 4
#define KV_OPT_PRODUCER_LANES 5
#define KV_OPT_HEAD_GROUP 6
#define KV_OPT_ITEM_COST 7
#define KV_OPT_PREFILL_PATH 8
#define KV_OPT_TEST_DROP_LOAD 9
#define KV_OPT_TEST_SLOW_SOFTMAX 10
#define KV_OPT_OUT_F32 11
#define KV_OPT_L2_POLICY 12
#define KV_OPT_EARLY_LOADS 13
KV_API kv_status kv_decode_set_option(int key, int value);
KV_API int kv_decode_get_option(int key);

/* ------------------------------------------------------------------------ */
/* Host block pool ("Module 23: Serving", 23.4; "Designing an LLM serving    */
/* system", "Paged attention" and "Caching and shortcuts": prefix caching)   */
/* ------------------------------------------------------------------------ */
/*
 * An opaque host object tracking which of num_blocks physical blocks are free
 * and how many sequences reference each used block. It owns no device memory.
 * Calls on one pool are serialised by an internal mutex.
 */
KV_API kv_status kv_pool_create(int num_blocks, void **pool_out);
KV_API void kv_pool_destroy(void *pool);

/* n fresh blocks (refcount 1 each) into ids_out[0..n), or KV_ERR_OOM with no
 * change if fewer than n are free. */
KV_API kv_status kv_pool_alloc(void *pool, int n, int32_t *ids_out);

/* One more reference to each listed block (a sequence sharing a prefix).
 * KV_ERR_STATE, with no change, if any listed block is free or out of range. */
KV_API kv_status kv_pool_incref(void *pool, const int32_t *ids, int n);

/* Drop one reference per listed entry; a block whose count reaches 0 becomes
 * free. KV_ERR_STATE, with no change, if that would take any count below 0. */
KV_API kv_status kv_pool_free(void *pool, const int32_t *ids, int n);

KV_API int kv_pool_num_free(const void *pool);
KV_API int kv_pool_num_blocks(const void *pool);
/* Reference count of block id, or -1 if id is out of range. */
KV_API int kv_pool_refcount(const void *pool, int32_t id);

/*
 * Host bookkeeping for one decode step of B sequences (host arrays):
 * sequence b currently caches context_lens[b] = c tokens; its new token goes
 * to position c. If c % 16 == 0 a fresh block is allocated and stored at
 * block_tables[b*W + c/16]. slot_mapping_out[b] = block*16 + c%16, and
 * context_lens[b] becomes c + 1. All or nothing: KV_ERR_OOM if the pool lacks
 * the blocks, KV_ERR_ARG if a sequence would exceed W blocks, KV_ERR_STATE if
 * the new token would land in a block shared with another sequence (refcount
 * > 1; copy-on-write is the caller's job). Nothing changes on error.
 * Afterwards each sequence holds exactly ceil(c'/16) blocks.
 */
KV_API kv_status kv_pool_append_slots(void *pool, int32_t *block_tables, int W,
                               int32_t *context_lens, int B,
                               int64_t *slot_mapping_out);

/*
 * Fork: child_row[i] = parent_row[i] for i < n_blocks, each block gaining one
 * reference (a child sequence starts on its parent's blocks, e.g. several
 * samples of one prompt). Host arrays; child_row may equal parent_row.
 * KV_ERR_STATE (nothing changed) if any id is out of range or free.
 */
KV_API kv_status kv_pool_fork(void *pool, const int32_t *parent_row, int n_blocks, int32_t *child_row);

/*
 * Copy-on-write variant of kv_pool_append_slots: when a sequence's new token
 * would land in a partly filled block that other sequences also reference,
 * the sequence gets a fresh block instead, the shared block loses that
 * reference, and the pair (shared block, fresh block) is written to
 * copy_src_out / copy_dst_out (host arrays of B entries; *n_copies_out is set).
 * Before this step's append, the caller copies every pair in every layer's K
 * and V cache (kv_cache_copy_blocks). If all sequences referencing a shared
 * block append to it in the same step, the last of them keeps the block.
 * ("Designing an LLM serving system", section "Paged attention": when
 * sequences sharing a block diverge, the block is copied on write.)
 * All or nothing: KV_ERR_OOM / KV_ERR_ARG / KV_ERR_STATE as kv_pool_append_slots.
 */
KV_API kv_status kv_pool_append_slots_cow(void *pool, int32_t *block_tables, int W,
                                          int32_t *context_lens, int B,
                                          int64_t *slot_mapping_out,
                                          int32_t *copy_src_out, int32_t *copy_dst_out,
                                          int *n_copies_out);

/* ------------------------------------------------------------------------ */
/* Whole-block moves over a list of cache tensors                            */
/* ------------------------------------------------------------------------ */
/*
 * caches is a HOST array of n_caches device pointers (1 <= n_caches <= 128;
 * n_caches == 0 or n == 0 is a no-op), each a cache tensor [num_blocks][16]
 * [Hkv][D] of element type dtype (KV_DTYPE_BF16 or KV_DTYPE_FP16; bytes are
 * moved as they are), typically every layer's K and V cache, so that one launch
 * serves a whole step. Block ids are device int32 arrays of n entries; an id
 * outside [0, num_blocks) is skipped and KV_STATUS_BAD_BLOCK_ID OR-ed into
 * *error_flag (device int32, may be NULL). All device pointers 16-byte aligned
 * (else KV_ERR_ARG); D a multiple of 8. Asynchronous on stream; nothing is
 * allocated.
 */
/*
 * Copy-on-write: caches[c][dst_ids[i]] = caches[c][src_ids[i]] for every c and
 * i < n. Destinations must be distinct and no block may be both a source and a
 * destination in one call (copies run in parallel). ("Designing an LLM serving
 * system", section "Paged attention": when sequences sharing a block diverge,
 * the block is copied on write.)
 */
KV_API kv_status kv_cache_copy_blocks(void *const *caches, int n_caches, const int32_t *src_ids,
                                      const int32_t *dst_ids, int n, int num_blocks, int Hkv, int D,
                                      int dtype, int32_t *error_flag, kv_stream_t stream);
/*
 * Swap-out staging: out[c][i] = caches[c][block_ids[i]], out a contiguous
 * device buffer [n_caches][n][16][Hkv][D] (then one device-to-host copy).
 * ("Designing an LLM serving system", section "Scheduling: when prefill meets
 * decode": under memory pressure a preempted sequence's cache blocks are
 * swapped out, and back in when it resumes.)
 */
KV_API kv_status kv_cache_gather_blocks(void *out, void *const *caches, int n_caches,
                                        const int32_t *block_ids, int n, int num_blocks, int Hkv,
                                        int D, int dtype, int32_t *error_flag, kv_stream_t stream);
/* Swap-in: caches[c][block_ids[i]] = in[c][i], in laid out as gather's out.
 * Ids must be distinct. */
KV_API kv_status kv_cache_scatter_blocks(void *const *caches, int n_caches, const void *in,
                                         const int32_t *block_ids, int n, int num_blocks, int Hkv,
                                         int D, int dtype, int32_t *error_flag, kv_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
