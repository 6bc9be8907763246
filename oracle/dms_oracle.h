/*
 * dms_oracle.h - plain, slow CPU oracle for the DMS decode path.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load this. The product library never links it,
 * and it shares no code, header or constant with the CUDA path.
 *
 * What it follows ("Inference-Time Hyper-Scaling with KV Cache Compression",
 * paper summary, Method and Key claims; sections 3.2 and 5.3, Fig. 5):
 *   - each KV head takes a binary eviction decision alpha_t for the token
 *     appended at step t;
 *   - a token marked at step t stays attendable until the window of w
 *     steps has passed, then leaves the cache (delayed eviction);
 *   - eviction acts as an additive mask on attention, which the oracle
 *     applies position by position.
 * Reading of the window bound: position j is visible to the query at step
 * s (j <= s) iff alpha_j == 0 or s - j < w.
 *
 * All arithmetic is in double precision.
 */
#ifndef DMS_ORACLE_H
#define DMS_ORACLE_H

#ifdef __cplusplus
extern "C" {
#endif

/* 1 if position j is attendable by the query of step s, else 0. */
int dmso_visible(long s, long j, int alpha_j, int window);

/* Masked softmax attention of g query heads over one KV stream, definition
 * form. K, V: [T][d] rows for positions 0..T-1 (T = s+1, the query sits at
 * position s). alpha: [T]. q: [g][d]. out: [g][d].
 * out[h] = sum_{j visible} softmax_j(scale * q[h].K[j]) V[j].
 * Writes zeros if no position is visible (T == 0). */
void dmso_attention(int T, int window, int d, int g, const double* q,
                    const double* K, const double* V, const unsigned char* alpha,
                    double scale, double* out);

/* Same as dmso_attention for n independent streams, run with OpenMP over
 * (stream, head) when built with it. Arrays of per-stream pointers. Returns
 * the number of threads used. */
int dmso_attention_batch(int n, const int* T, int window, int d, int g,
                         const double* const* q, const double* const* K,
                         const double* const* V, const unsigned char* const* alpha,
                         double scale, double* const* out);

/* ---- slot-pool simulator (the build's allocation policy, sequential) ----
 * Stream id = seq * num_kv_heads + kv_head. Each stream keeps n logical
 * slots [0, n), mapped to physical slots through its page table
 * (page_size slots per page). Pages come from one global free stack whose
 * pops return 0, 1, 2, ... from a fresh pool.
 * Appending token s to a stream: if s >= w and the token at s - w was
 * marked (alpha = 1), it leaves now and s takes its logical slot; otherwise
 * s takes the fresh logical slot n (a new page is popped first when n is a
 * multiple of page_size) and n grows by one.
 * Streams of one append call go in (sequence order of the call, KV head
 * ascending) order; all tokens of a stream go before the next stream. */
typedef struct dmso_sim dmso_sim;

enum { DMSO_OK = 0, DMSO_ERR_INVALID = 1, DMSO_ERR_POOL_EXHAUSTED = 2,
       DMSO_ERR_STREAM_FULL = 6 };

dmso_sim* dmso_sim_create(int max_seqs, int num_kv_heads, int window, int page_size,
                          int max_pages, int max_pages_per_stream);
void dmso_sim_destroy(dmso_sim* sim);

/* counts[i] tokens for seq_ids[i]; alpha is [sum(counts)][num_kv_heads] in
 * call order. If phys_slot is not NULL it receives the physical slot of
 * every appended (token, kv head), same layout as alpha. */
int dmso_sim_append(dmso_sim* sim, int n_seqs, const int* seq_ids, const int* counts,
                    const unsigned char* alpha, int* phys_slot);

/* Return every page of the sequence to the free stack (KV heads ascending,
 * each stream's pages last to first) and clear its streams. */
int dmso_sim_reset_seq(dmso_sim* sim, int seq_id);

/* Copy out the state. Any pointer may be NULL. page_table: [S][mps] (-1 for
 * unused), n_pages/n/pos: [S], slot_pos: [max_pages*page_size] (-1 for a
 * never-written slot), free_list: [max_pages], free_count: [1]. */
void dmso_sim_snapshot(const dmso_sim* sim, int* page_table, int* n_pages, int* n, int* pos,
                       int* slot_pos, int* free_list, int* free_count);

/* Positions held by the logical slots [0, n) of one stream, in slot order.
 * Returns n. */
int dmso_sim_retained(const dmso_sim* sim, int stream, int* positions);

#ifdef __cplusplus
}
#endif
#endif
