/*
 * dms.h - C ABI of libdms: decode-time Dynamic Memory Sparsification (DMS)
 * over a paged, per-KV-head slot pool on one NVIDIA B200 (sm_100a).
 *
 * The method ("Inference-Time Hyper-Scaling with KV Cache Compression",
 * paper summary, Key claims and Method, section 3.2):
 *   - every KV head takes a binary eviction decision alpha_t for the token
 *     it appends at step t;
 *   - delayed eviction: a token marked at step t stays attendable until
 *     step t + w (w = 256 by default, section 5.3 and Fig. 5), then leaves;
 *   - eviction acts as an attention mask that is never materialised, and the
 *     sparsified cache works with paged KV storage (section 3.2
 *     "Performance Considerations", section 3.3).
 * Reading of the window bound used throughout: position j is visible to
 * the query at step s iff alpha_j == 0 or s - j < w.
 *
 * The pages define the computation, not an API. Each call below names the
 * passage it serves; the cache life-cycle and inspection calls, for which
 * the pages define nothing, say so.
 *
 * Storage. A *stream* is one (sequence, KV head) pair, stream id =
 * seq_id * num_kv_heads + kv_head. A stream holds its retained tokens in
 * logical slots [0, n); logical slot l lives in physical page
 * page_table[stream][l / 16] at row l % 16. A page holds 16 K rows then 16
 * V rows of head_dim elements each, contiguous. Pages come from one global
 * free stack (a fresh pool pops 0, 1, 2, ...).
 * When token s is appended to a stream and s >= w and the token at s - w
 * was marked, that token leaves now and s takes its logical slot; otherwise
 * s takes the fresh slot n and n grows by one, popping a page first when n
 * is a multiple of 16. Hence slots [0, n) are always exactly the retained
 * tokens and n never shrinks while a sequence lives.
 * Within one append call, streams take pages in (order of seq_ids in the
 * call, KV head ascending) order.
 *
 * Conventions.
 *   - Every tensor argument is caller-owned DEVICE memory on the cache's
 *     device, row-major and contiguous, unless stated otherwise.
 *   - Calls enqueue work on the caller's stream and return without
 *     synchronising, except where stated ("syncs").
 *   - Errors found on the host (bad arguments, CUDA launch failures) are
 *     returned at once. Errors found on the device (pool exhausted, stream
 *     full, bad sequence id, bounded-wait timeout) latch into a status word
 *     and *poison* the cache: every later kernel on it does nothing until
 *     dms_cache_reset. Read the word with dms_get_status (syncs).
 *   - One cache must not be used from two streams at the same time. Calls
 *     on one cache run in the order they are made: on one stream, or on
 *     streams ordered by events. dms_append of a step must precede the
 *     dms_decode_attention that should see that step's token.
 *   - Different caches may be used from different streams at the same
 *     time, in any interleaving. No kernel of this library waits on another
 *     of its CTAs, so a launch finishes with whatever share of the SMs it
 *     gets, however the device is shared.
 *   - seq_ids inside one call must be distinct.
 */
#ifndef DMS_H
#define DMS_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct dms_cache dms_cache;   /* opaque, owned by the library */

typedef enum {
    DMS_OK = 0,
    DMS_ERR_INVALID = 1,          /* bad argument or configuration */
    DMS_ERR_POOL_EXHAUSTED = 2,   /* free page stack empty (device) */
    DMS_ERR_CUDA = 3,             /* a CUDA call failed */
    DMS_ERR_TIMEOUT = 4,          /* a bounded wait inside a kernel ran out (device) */
    DMS_ERR_POISONED = 5,         /* host calls refuse work once dms_get_status saw a device error */
    DMS_ERR_STREAM_FULL = 6,      /* a stream would exceed max_pages_per_stream (device) */
    DMS_ERR_BAD_SEQ = 7           /* a device-side seq_id outside [0, max_seqs) (device) */
} dms_status;

typedef enum { DMS_BF16 = 0, DMS_F32 = 1 } dms_dtype;

typedef enum {
    DMS_ATTN_AUTO = 0,   /* tensor-core page kernel for bf16, CUDA-core kernel for f32 */
    DMS_ATTN_SIMT = 1,   /* CUDA-core kernel: warp-shuffle dot products, any dtype */
    DMS_ATTN_MMA = 2     /* mma.sync m16n8k16 page kernel (bf16 only, GQA group <= 8) */
} dms_attn_kernel;

typedef struct {
    int32_t max_seqs;              /* sequences the cache can hold (seq_id in [0, max_seqs)) */
    int32_t num_kv_heads;          /* KV heads per sequence; max_seqs * num_kv_heads <= 8192 */
    int32_t head_dim;              /* 64 or 128 */
    int32_t page_size;             /* must be 16 */
    int32_t window;                /* delayed-eviction window w >= 1 */
    int32_t max_pages;             /* pages in the shared pool, 1 .. 2^27 */
    int32_t max_pages_per_stream;  /* page-table length of one stream */
    dms_dtype dtype;               /* storage type of K, V (and Q) */
    dms_attn_kernel attn_kernel;   /* decode-attention kernel choice */
} dms_config;

/* Create a cache on the current CUDA device (life cycle; the pages define no
 * API: they fix only that the cache is paged and per head, section 3.2
 * "Performance Considerations"). Allocates the pool
 * (max_pages * 2 * 16 * head_dim elements), the page tables, the free stack,
 * the per-stream counters and window rings, and the split-K scratch
 * (partials and per-stream counters). Zeroes everything. Syncs.
 * Returns DMS_ERR_INVALID for an unsupported configuration, DMS_ERR_CUDA if
 * an allocation fails (nothing leaks). */
dms_status dms_cache_create(const dms_config* cfg, dms_cache** out);

/* Free everything (life cycle; the pages define no API). Syncs the device.
 * NULL is accepted. */
dms_status dms_cache_destroy(dms_cache* cache);

/* Return the cache to its freshly created state: all sequences empty, free
 * stack full, status cleared (life cycle; the pages define no API). Pool
 * contents are not cleared. Async. */
dms_status dms_cache_reset(dms_cache* cache, cudaStream_t stream);

/* Release sequence seq_id (host int): push its pages back on the free stack
 * (KV head ascending, each stream's pages last to first) and clear its
 * counters and window rings (life cycle; the pages define no API). Async. */
dms_status dms_seq_reset(dms_cache* cache, cudaStream_t stream, int32_t seq_id);

/* Append tokens and apply delayed eviction (paper summary, Method; section
 * 3.2: the decision taken at step t acts at step t + w). For every
 * (sequence, KV head) stream of the call and every new token s in position
 * order: retire the token at s - w if it was marked and reuse its slot, else
 * take a fresh slot; write the K and V rows into the pool; record alpha_s.
 *   n_seqs        sequences in this call (host int, >= 0)
 *   seq_ids       device int32 [n_seqs], distinct, each in [0, max_seqs)
 *   cu_tokens     device int32 [n_seqs + 1] prefix offsets of each
 *                 sequence's tokens, or NULL for exactly one token per
 *                 sequence (the decode step; total_tokens must be n_seqs)
 *   total_tokens  host int, rows in K, V and alpha
 *   K, V          device [total_tokens, num_kv_heads, head_dim] of dtype;
 *                 rows of sequence i are cu_tokens[i] .. cu_tokens[i+1]-1
 *   alpha         device uint8 [total_tokens, num_kv_heads]; 0 keeps the
 *                 token, any other value marks it for delayed eviction
 * Device errors: DMS_ERR_POOL_EXHAUSTED (no page is taken by any stream
 * that needed one in this call; those streams are left unchanged),
 * DMS_ERR_STREAM_FULL, DMS_ERR_BAD_SEQ. Async. */
dms_status dms_append(dms_cache* cache, cudaStream_t stream, int32_t n_seqs,
                      const int32_t* seq_ids, const int32_t* cu_tokens, int32_t total_tokens,
                      const void* K, const void* V, const uint8_t* alpha);

/* dms_append with the eviction decisions read from the keys (paper summary,
 * Method: one neuron of the K projection per head is repurposed to give the
 * eviction logit). The pages do not say how the logit is binarised at
 * inference; the library takes alpha = 1 iff the logit is > 0. For every
 * appended token t and KV head h: alpha = 1 iff K[t, h, alpha_channel] > 0
 * (zero and NaN keep the token). K and V are stored as given, the logit
 * channel included. Same bookkeeping and errors as dms_append with those
 * alpha bits.
 *   alpha_channel  host int in [0, head_dim) */
dms_status dms_append_keyed(dms_cache* cache, cudaStream_t stream, int32_t n_seqs, const int32_t* seq_ids,
                            const int32_t* cu_tokens, int32_t total_tokens, const void* K, const void* V,
                            int32_t alpha_channel);

/* Eviction decisions from a designated logit channel of a projection (paper
 * summary, Method: one neuron of the K or the Q projection per head is
 * repurposed to give the eviction logit; taken as alpha = 1 iff the logit is
 * > 0, zero and NaN keep the token). Needs no cache.
 *   X             device [rows, num_kv_heads * heads_per_kv, head_dim] of
 *                 dtype: keys (heads_per_kv = 1) or queries (heads_per_kv =
 *                 g, the GQA group; query heads k*g .. k*g+g-1 belong to KV
 *                 head k)
 *   head          host int in [0, heads_per_kv): the designated head of
 *                 each KV head's group (0 for keys)
 *   channel       host int in [0, head_dim)
 *   alpha_out     device uint8 [rows, num_kv_heads]:
 *                 alpha_out[r, k] = X[r, k * heads_per_kv + head, channel] > 0
 * The result feeds dms_append's alpha argument. Async. */
dms_status dms_alpha_from_logit(cudaStream_t stream, const void* X, dms_dtype dtype, int32_t rows,
                                int32_t num_kv_heads, int32_t heads_per_kv, int32_t head, int32_t head_dim,
                                int32_t channel, uint8_t* alpha_out);

/* One decode step of GQA attention over the retained tokens (paper summary,
 * Key claims: memory reads dominate decode latency; the mask is never
 * materialised). For each sequence b of the call and query head h:
 *   out[b, h] = sum_{j retained} softmax_j(scale * Q[b, h] . K_j) V_j
 * over the retained tokens of stream (seq_ids[b], h / g), g = num_q_heads /
 * num_kv_heads. Split-K over retained pages with fp32 online softmax; the
 * partial results are merged inside the same kernel (no second launch).
 *   seq_ids      device int32 [n_seqs], distinct
 *   Q            device [n_seqs, num_q_heads, head_dim] of the cache dtype
 *   num_q_heads  host int; a multiple of num_kv_heads with g <= 8
 *   scale        host float (usually 1 / sqrt(head_dim))
 *   out          device [n_seqs, num_q_heads, head_dim] of out_dtype
 * A stream with no tokens yields zeros.
 * Each call leaves its stream list on the device for the next call on the
 * cache. When the kernel just before a call in its stream is not one of this
 * cache's, the call guesses that it has the previous call's streams. It plans
 * from the cache state and starts its first page copies before that kernel has
 * finished (programmatic dependent launch), and checks the guess against
 * seq_ids once it has. Async. */
dms_status dms_decode_attention(dms_cache* cache, cudaStream_t stream, int32_t n_seqs,
                                const int32_t* seq_ids, const void* Q, int32_t num_q_heads,
                                float scale, void* out, dms_dtype out_dtype);

/* One whole decode step in one launch: dms_append of one token per sequence
 * (cu_tokens = NULL) followed by dms_decode_attention, with the same results:
 * the same bookkeeping bit for bit, and outputs equal up to fp32 rounding
 * order (paper summary, Key claims: decode is bound by memory reads and DMS
 * adds no read or write of the KV cache, so the step should cost one pass
 * over the retained K/V and one launch).
 * The attention runs over the cache as it was before the step, with the row
 * of the token that leaves at this step masked and the new token taken
 * from K and V; the append's writes go to rows that no part of the launch
 * attends. The launch reads one copy of the per-stream counts and writes
 * the other (the cache keeps two and flips between them), so none of its
 * CTAs waits on another. A cache with more than 1024 streams (max_seqs *
 * num_kv_heads), or whose configuration leaves no shared memory for the
 * step's per-stream state, issues the two launches instead; so does a call
 * on a stream that is being captured into a CUDA graph (the fused launch
 * carries host sequence numbers and cannot be replayed).
 * Each fused step leaves the next one on the same cache a schedule: every
 * call stream's count, position and leaving slot after it, and the page ids
 * of every CTA's range. The next fused step uses it when no other call has
 * changed the cache in between (it checks the entries against its seq ids
 * and falls back stream by stream), which saves it two dependent memory
 * round trips. When, in addition, the kernel just before it in the stream is
 * not one of this cache's, it plans and starts its first page copies before
 * that kernel has finished (programmatic dependent launch), on the guess that
 * its seq ids are those of the step that left the schedule; the guess is
 * checked once the previous kernel is done.
 * Every kernel of this library that writes a cache lets the next kernel of its
 * stream start only after its own dependency wait; other code that uses
 * programmatic dependent launch on the same stream must do the same (call
 * cudaGridDependencySynchronize before cudaTriggerProgrammaticLaunchCompletion).
 *   n_seqs, seq_ids      as dms_append (one token per sequence)
 *   K, V                 device [n_seqs, num_kv_heads, head_dim] of the cache dtype, 16-B aligned
 *   alpha                device uint8 [n_seqs, num_kv_heads]
 *   Q, num_q_heads, scale, out, out_dtype   as dms_decode_attention
 * Device errors latch as in dms_append (pool exhausted, stream full, bad
 * seq id); the outputs of that launch are then unspecified. Async. */
dms_status dms_decode_step(dms_cache* cache, cudaStream_t stream, int32_t n_seqs, const int32_t* seq_ids,
                           const void* K, const void* V, const uint8_t* alpha, const void* Q,
                           int32_t num_q_heads, float scale, void* out, dms_dtype out_dtype);

/* dms_decode_step with the eviction decisions read from the keys, as
 * dms_append_keyed: alpha = 1 iff K[b, h, alpha_channel] > 0 (paper summary,
 * Method: a repurposed K neuron gives the logit). */
dms_status dms_decode_step_keyed(dms_cache* cache, cudaStream_t stream, int32_t n_seqs, const int32_t* seq_ids,
                                 const void* K, const void* V, int32_t alpha_channel, const void* Q,
                                 int32_t num_q_heads, float scale, void* out, dms_dtype out_dtype);

/* dms_decode_step with the eviction decisions read from the step's queries
 * (paper summary, Method: the repurposed neuron may come from the Q
 * projection instead). The decision of KV head k is taken from query head
 * k * g + alpha_head (the designated head of its group):
 * alpha = 1 iff Q[b, k * g + alpha_head, alpha_channel] > 0.
 *   alpha_head     host int in [0, g)
 *   alpha_channel  host int in [0, head_dim) */
dms_status dms_decode_step_qkeyed(dms_cache* cache, cudaStream_t stream, int32_t n_seqs, const int32_t* seq_ids,
                                  const void* K, const void* V, const void* Q, int32_t num_q_heads,
                                  int32_t alpha_head, int32_t alpha_channel, float scale, void* out,
                                  dms_dtype out_dtype);

/* Retained counts and compression ratios (paper summary, Key claims: CR =
 * tokens seen / tokens kept; each head can land at its own CR). Async;
 * every output is device memory and optional (NULL skips it).
 *   retained  int32 [max_seqs * num_kv_heads]  n of every stream
 *   seen      int32 [max_seqs * num_kv_heads]  tokens appended to every stream
 *   head_cr   float [num_kv_heads]   sum(seen) / sum(retained) over all
 *             sequences for each KV head (0 when nothing is retained)
 *   totals    int64 [2]              { sum(seen), sum(retained) } */
dms_status dms_stats(dms_cache* cache, cudaStream_t stream, int32_t* retained, int32_t* seen,
                     float* head_cr, int64_t* totals);

/* dms_stats with HOST outputs (paper summary, Key claims, as dms_stats).
 * Syncs the stream. Any pointer may be NULL.
 *   retained, seen  host int32 [max_seqs * num_kv_heads], as dms_stats
 *   cr_overall      host double: sum(seen) / sum(retained) over every
 *                   stream (0 when nothing is retained) */
dms_status dms_stats_host(dms_cache* cache, cudaStream_t stream, int32_t* retained, int32_t* seen,
                          double* cr_overall);

/* Copy the bookkeeping to HOST memory for checking (inspection; the pages
 * define no API). Syncs the stream. Any pointer may be NULL.
 *   page_table  int32 [S * max_pages_per_stream]   (entries >= n_pages are stale)
 *   n_pages, n, pos  int32 [S]
 *   slot_pos    int32 [max_pages * 16]  position stored in each physical slot
 *               (stale outside a stream's slots [0, n))
 *   free_list   int32 [max_pages], free_count int32 [1] */
dms_status dms_snapshot(dms_cache* cache, cudaStream_t stream, int32_t* page_table,
                        int32_t* n_pages, int32_t* n, int32_t* pos, int32_t* slot_pos,
                        int32_t* free_list, int32_t* free_count);

/* Gather the retained K and V rows of one stream in logical slot order into
 * device buffers [n, head_dim] of the cache dtype (inspection; the pages
 * define no API). n from dms_stats or dms_snapshot; rows_cap bounds the
 * copy. Async. */
dms_status dms_gather_kv(dms_cache* cache, cudaStream_t stream, int32_t seq_id,
                         int32_t kv_head, int32_t rows_cap, void* K_out, void* V_out);

/* ---- Decode attention that allocates nothing ---------------------------
 * The paper has no counterpart to this call. It is for callers that must
 * not allocate device memory while they decode: a framework whose caching
 * allocator already holds the device memory (a cudaMalloc of its own could
 * fail or synchronise the device), or a runtime that owns every buffer and
 * lends the library its K/V pages. dms_decode_attention cannot serve them,
 * because its scratch comes with a dms_cache, and dms_cache_create
 * allocates.
 *
 * Same arithmetic and kernels as dms_decode_attention, over K/V pages the
 * caller owns and lays out as a dms_cache does (see "Storage" above). The
 * split-K scratch (partials, arrival counters, status word) is a static
 * device array of about 4.1 MiB inside the library. The CUDA runtime
 * places it on each device that loads the library and keeps it until the
 * process exits. The call itself makes no cudaMalloc, cudaFree or other
 * allocating call.
 *
 * The first call on a device (with that device current) looks up the
 * array's device address and sets the kernel's attributes. Make that first
 * call before any stream capture. Later calls reuse the set-up; the launch
 * plans of the last 8 distinct call shapes (pool, head_dim, dtype, streams,
 * max_pages) are kept, so alternating shapes prepare nothing again.
 *
 * Every call on a device shares the one array: calls whose kernels may
 * overlap on the GPU (different streams, no ordering between them) race on
 * it and give wrong results. Each call clears the counters and status word
 * it uses on `stream` (cudaMemsetAsync) before its kernel.
 *
 * Limits: n_seqs * num_kv_heads <= DMS_NOALLOC_MAX_STREAMS, and the grid
 * (one CTA per SM) plus the streams <= DMS_NOALLOC_MAX_PIECES. Beyond them
 * the call returns DMS_ERR_INVALID and launches nothing.
 *
 *   kv           host pointer to the description of the caller's cache:
 *     kv_pool      device [max_pages][2][16][head_dim] of dtype, 16-B aligned:
 *                  per page 16 K rows then 16 V rows
 *     page_table   device int32 [max_seqs * num_kv_heads][max_pages_per_stream]
 *     retained     device int32 [max_seqs * num_kv_heads]: n of each stream;
 *                  its tokens sit in logical slots [0, n). A count outside
 *                  [0, 16 * max_pages_per_stream] is clamped into it: a larger
 *                  one attends every slot the page table addresses, a negative
 *                  one attends nothing (zeros out).
 *   seq_ids, Q, num_q_heads, scale, out, out_dtype: as dms_decode_attention.
 * Device-side checks (a seq id outside [0, max_seqs), a page id outside
 * [0, max_pages), a clamped count) skip or bound the bad access, but no
 * later call reports them: the outputs of those streams are then
 * unspecified, except as the clamp above states. Async. */
#define DMS_NOALLOC_MAX_STREAMS 512
#define DMS_NOALLOC_MAX_PIECES 1024

typedef struct {
    const void* kv_pool;
    const int32_t* page_table;
    const int32_t* retained;
    int32_t max_seqs;
    int32_t num_kv_heads;
    int32_t head_dim;              /* 64 or 128 */
    int32_t max_pages;
    int32_t max_pages_per_stream;
    dms_dtype dtype;               /* storage type of K, V and Q */
} dms_paged_kv;

dms_status dms_decode_attention_noalloc(cudaStream_t stream, const dms_paged_kv* kv, int32_t n_seqs,
                                        const int32_t* seq_ids, const void* Q, int32_t num_q_heads,
                                        float scale, void* out, dms_dtype out_dtype);

/* Sync the stream and return the latched device status, DMS_OK if none
 * (failure detection; the pages define no API). */
dms_status dms_get_status(dms_cache* cache, cudaStream_t stream);

/* Static description of a status code. */
const char* dms_status_string(dms_status s);

/* Failure-detection self-test (no counterpart in the paper): one block runs
 * the library's two bounded waits on conditions that never come true.
 *  1. a spin on a flag that nothing sets;
 *  2. an mbarrier phase whose expected bytes never arrive (afterwards the
 *     block completes that phase itself, so nothing is pending at exit).
 * Each gives up after about 2^31 SM cycles (about a second), latches
 * DMS_ERR_TIMEOUT into the cache's status word and returns. No fault, trap or
 * hang. The cache is then poisoned as by any device error: dms_get_status
 * returns DMS_ERR_TIMEOUT, and work-issuing calls are refused until
 * dms_cache_reset.
 *   timed_out  device int32 [2]: 1 where each wait gave up, else 0
 * Async. */
dms_status dms_selftest_bounded_waits(dms_cache* cache, cudaStream_t stream, int32_t* timed_out);

/* Kernel launches issued by the library since the cache was created (host
 * counter, for accounting; the pages define no API). */
int64_t dms_launch_count(const dms_cache* cache);

#ifdef __cplusplus
}
#endif
#endif /* DMS_H */
