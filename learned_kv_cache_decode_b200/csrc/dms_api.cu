// dms_api.cu - the extern "C" boundary of libdms (see include/dms.h).
//
// Host code only: argument checks, allocation, and kernel launches on the
// caller's stream. Every step of the decode path runs in the kernels of
// dms_append.cu and dms_attention.cu.
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <new>
#include <thread>

#include <nvtx3/nvToolsExt.h>

#include "dms_internal.cuh"

struct dms_cache {
  dms_config cfg;
  int device = 0;
  int num_sms = 0;
  dms::Dev dv{};
  dms::AttnPlan plan{};
  dms::AttnPlan step_plan{};   // fused decode step (append + attention in one launch)
  bool has_step = false;       // else dms_decode_step issues the two launches
  // State parity after every launch issued so far (see dms::kCtrlPar): it flips
  // with every fused step, the only kernel that changes it. Eager launches take
  // it from here; a launch into a stream under capture reads the device word.
  int par = 0;
  // Schedules fused steps leave for the next one (see dms::NextPlan): the tag of
  // the last fused launch, and the tag the next fused launch may trust (0 once
  // any other call has changed the cache).
  dms::NextPlan next{};
  uint64_t step_tags = 0;
  uint64_t trust_tag = 0;
  // Stream lists of the last attention calls ([2][1 + max_seqs], see dms::AttnGuess)
  // and the number of attention launches so far (its parity picks the buffers).
  int32_t* attn_guess = nullptr;
  uint64_t attn_launches = 0;
  int64_t* totals_dev = nullptr;   // {sum(seen), sum(retained)} for dms_stats_host
  int64_t launches = 0;
  bool poisoned = false;   // a device error was observed by dms_get_status
};

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// An NVTX range named after the API call, for profiler timelines (a no-op
// unless a tool is attached).
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};

// The cache whose kernels were launched last on each stream. Kernels that
// write a cache are launched only through these calls, and each lets the next
// kernel of its stream start only after its own dependency wait. So when the
// record of a stream names another cache, no kernel still running ahead of the
// next launch on that stream writes this one. The stats kernel, which writes
// no cache state and lets the next kernel start at once, is not recorded. A
// stream with no record, or one whose record was evicted, counts as this
// cache's. The per-thread default stream is a different stream in every host
// thread.
struct StreamLast {
  int device;
  cudaStream_t stream;
  std::thread::id thread;
  const dms_cache* cache;
};
constexpr int kStreamRecords = 64;
std::mutex g_last_mu;
StreamLast g_last[kStreamRecords];
int g_last_next = 0;

// Records `c` as the last cache launched on `s`; returns true when the
// previous record of `s` named another cache. A launch into a stream being
// captured into a graph runs later, if at all, so it is neither recorded nor
// started early (a graph launch waits for the work before it in its stream).
bool note_launch(const dms_cache* c, int device, cudaStream_t s) {
  cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &capture) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (capture != cudaStreamCaptureStatusNone) return false;
  const std::thread::id th = s == cudaStreamPerThread ? std::this_thread::get_id() : std::thread::id();
  std::lock_guard<std::mutex> lock(g_last_mu);
  for (StreamLast& e : g_last) {
    if (e.cache && e.device == device && e.stream == s && e.thread == th) {
      const bool other = e.cache != c;
      e.cache = c;
      return other;
    }
  }
  g_last[g_last_next] = StreamLast{device, s, th, c};
  g_last_next = (g_last_next + 1) % kStreamRecords;
  return false;
}

dms_status from_cuda(cudaError_t e) { return e == cudaSuccess ? DMS_OK : DMS_ERR_CUDA; }

// Whether `s` is being captured into a CUDA graph (-1: the query failed).
int capturing(cudaStream_t s) {
  cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &capture) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  return capture != cudaStreamCaptureStatusNone ? 1 : 0;
}

// Retained counts for an attention launch of this cache on `s`.
dms::AttnCounts counts_for(const dms_cache* h, cudaStream_t s) {
  return dms::AttnCounts{h->dv.n, h->dv.S, capturing(s) == 0 ? h->par : -1};
}

// Where an append or a fused step takes its eviction decisions from.
dms::AlphaSrc alpha_src(const dms_cache* h, const void* K, const void* Q, int hq, const dms::AlphaChoice& c) {
  const dms::Dev& dv = h->dv;
  if (c.channel < 0) return dms::alpha_given(c.alpha, dv.hkv);
  if (c.q_head < 0) return dms::alpha_from_keys(K, dv.hkv, dv.d, c.channel, dv.elem_bytes);
  return dms::alpha_from_queries(Q, dv.hkv, hq / dv.hkv, dv.d, c.q_head, c.channel, dv.elem_bytes);
}

// Every call must run with the cache's device current.
dms_status check_device(const dms_cache* c) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return DMS_ERR_CUDA;
  return dev == c->device ? DMS_OK : DMS_ERR_INVALID;
}

// Work-issuing calls refuse a cache whose device error has been observed.
dms_status check_usable(const dms_cache* c) {
  if (dms_status s = check_device(c)) return s;
  return c->poisoned ? DMS_ERR_POISONED : DMS_OK;
}

void free_all(dms::Dev& dv) {
  void* ptrs[] = {dv.pos, dv.n, dv.n_pages, dv.page_table, dv.ring, dv.slot_pos, dv.free_list,
                  dv.ctrl, dv.scratch, dv.kv, dv.part, dv.cnt};
  for (void* p : ptrs)
    if (p) cudaFree(p);
  dv = dms::Dev{};
}

template <typename T>
cudaError_t alloc(T** p, size_t count) {
  return cudaMalloc(reinterpret_cast<void**>(p), count * sizeof(T) + 16);
}

void free_next(dms::NextPlan& np) {
  void* ptrs[] = {np.entry, np.hdr, np.list};
  for (void* p : ptrs)
    if (p) cudaFree(p);
  np = dms::NextPlan{};
}

// Buffers of the schedules a fused step leaves for the next one: per tag
// parity, one entry per stream and one page list per CTA of the step's grid,
// long enough for any range (a call holds at most max_pages pages in at most
// S streams; a range spans at most 1 / grid of their weighted cost).
cudaError_t alloc_next(const dms::Dev& dv, int grid, dms::NextPlan* np) {
  np->cap = (int)std::max<int64_t>(
      1, ((int64_t)dv.max_pages + (int64_t)dms::kMaxPieceCost * dv.S + grid - 1) / grid);
  np->S = dv.S;
  cudaError_t e = alloc(&np->entry, (size_t)2 * dv.S);
  if (e == cudaSuccess) e = alloc(&np->hdr, (size_t)2 * grid * 2);
  if (e == cudaSuccess) e = alloc(&np->list, (size_t)2 * grid * np->cap);
  if (e == cudaSuccess) e = cudaMemset(np->entry, 0, (size_t)2 * dv.S * sizeof(dms::PlanEntry));
  if (e == cudaSuccess) e = cudaMemset(np->hdr, 0, (size_t)2 * grid * 2 * sizeof(int4));
  return e;
}

}  // namespace

extern "C" {

dms_status dms_cache_create(const dms_config* cfg, dms_cache** out) {
  const CallRange range("dms_cache_create");
  if (!cfg || !out) return DMS_ERR_INVALID;
  *out = nullptr;
  const dms_config& c = *cfg;
  if (c.max_seqs < 1 || c.num_kv_heads < 1 || c.num_kv_heads > dms::kMaxKvHeads) return DMS_ERR_INVALID;
  if ((int64_t)c.max_seqs * c.num_kv_heads > dms::kMaxStreams) return DMS_ERR_INVALID;
  if (c.head_dim != 64 && c.head_dim != 128) return DMS_ERR_INVALID;
  if (c.page_size != dms::kPage || c.window < 1) return DMS_ERR_INVALID;
  if (c.max_pages < 1 || c.max_pages > (1 << 27) || c.max_pages_per_stream < 1) return DMS_ERR_INVALID;
  if (c.dtype != DMS_BF16 && c.dtype != DMS_F32) return DMS_ERR_INVALID;
  if (c.attn_kernel != DMS_ATTN_AUTO && c.attn_kernel != DMS_ATTN_SIMT && c.attn_kernel != DMS_ATTN_MMA)
    return DMS_ERR_INVALID;
  if (c.attn_kernel == DMS_ATTN_MMA && c.dtype != DMS_BF16) return DMS_ERR_INVALID;
  if ((int64_t)c.max_seqs * c.num_kv_heads * ((int64_t)c.window + 1) > (int64_t)1 << 31) return DMS_ERR_INVALID;
  if ((int64_t)c.max_seqs * c.num_kv_heads * c.max_pages_per_stream > (int64_t)1 << 31) return DMS_ERR_INVALID;

  dms_cache* h = new (std::nothrow) dms_cache();
  if (!h) return DMS_ERR_CUDA;
  h->cfg = c;
  if (cudaGetDevice(&h->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess) {
    delete h;
    return DMS_ERR_CUDA;
  }
  dms::Dev& dv = h->dv;
  dv.S = c.max_seqs * c.num_kv_heads;
  dv.hkv = c.num_kv_heads;
  dv.d = c.head_dim;
  dv.w = c.window;
  dv.mps = c.max_pages_per_stream;
  dv.max_pages = c.max_pages;
  dv.max_seqs = c.max_seqs;
  dv.elem_bytes = c.dtype == DMS_BF16 ? 2 : 4;

  const size_t S = dv.S;
  cudaError_t e = cudaSuccess;
  auto step = [&](cudaError_t r) { if (e == cudaSuccess) e = r; };
  step(alloc(&dv.pos, 2 * S));   // one copy per state parity
  step(alloc(&dv.n, 2 * S));
  step(alloc(&dv.n_pages, S));
  step(alloc(&dv.page_table, S * dv.mps));
  step(alloc(&dv.ring, S * ((size_t)dv.w + 1)));
  step(alloc(&dv.slot_pos, (size_t)dv.max_pages * dms::kPage));
  step(alloc(&dv.free_list, (size_t)dv.max_pages));
  step(alloc(&dv.ctrl, (size_t)dms::kCtrlWords));
  step(alloc(&dv.scratch, S));
  step(alloc(&dv.cnt, S));
  step(alloc(&dv.kv, (size_t)dv.max_pages * 2 * dms::kPage * dv.d * dv.elem_bytes));
  if (e == cudaSuccess) e = dms::prepare_aux_kernels();
  if (e == cudaSuccess) e = dms::attention_prepare(dv, c.dtype, c.attn_kernel, h->num_sms, &h->plan);
  if (e == cudaSuccess && dv.S <= dms::kStepMaxStreams) {
    // The fused step needs its per-stream decisions in shared memory; a
    // configuration that leaves no room for them falls back to two launches.
    h->has_step = dms::step_prepare(dv, c.dtype, c.attn_kernel, h->num_sms, &h->step_plan) == cudaSuccess;
    cudaGetLastError();
  }
  if (e == cudaSuccess && h->has_step) e = alloc_next(dv, h->step_plan.grid, &h->next);
  if (e == cudaSuccess) e = alloc(&h->attn_guess, (size_t)2 * (1 + c.max_seqs));
  if (e == cudaSuccess) e = alloc(&h->totals_dev, (size_t)2);
  if (e == cudaSuccess) e = cudaMemset(h->attn_guess, 0xff, (size_t)2 * (1 + c.max_seqs) * sizeof(int32_t));
  const int grid = h->has_step && h->step_plan.grid > h->plan.grid ? h->step_plan.grid : h->plan.grid;
  dv.part_slots = grid + dv.S;
  if (e == cudaSuccess) e = alloc(&dv.part, ((size_t)grid + dv.S) * dms::kMaxGroup * (dv.d + 2));
  if (e == cudaSuccess) e = cudaMemset(dv.kv, 0, (size_t)dv.max_pages * 2 * dms::kPage * dv.d * dv.elem_bytes);
  if (e == cudaSuccess) e = cudaMemset(dv.page_table, 0xff, S * dv.mps * sizeof(int32_t));
  if (e == cudaSuccess) e = cudaMemset(dv.slot_pos, 0xff, (size_t)dv.max_pages * dms::kPage * sizeof(int32_t));
  if (e == cudaSuccess) e = dms::launch_init_state(dv, 0);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    free_all(dv);
    free_next(h->next);
    if (h->attn_guess) cudaFree(h->attn_guess);
    if (h->totals_dev) cudaFree(h->totals_dev);
    delete h;
    cudaGetLastError();
    return e == cudaErrorInvalidValue ? DMS_ERR_INVALID : DMS_ERR_CUDA;
  }
  h->launches = 1;
  *out = h;
  return DMS_OK;
}

dms_status dms_cache_destroy(dms_cache* h) {
  const CallRange range("dms_cache_destroy");
  if (!h) return DMS_OK;
  int prev = -1;
  cudaGetDevice(&prev);
  cudaSetDevice(h->device);
  cudaError_t e = cudaDeviceSynchronize();
  free_all(h->dv);
  free_next(h->next);
  if (h->attn_guess) cudaFree(h->attn_guess);
  if (h->totals_dev) cudaFree(h->totals_dev);
  if (prev >= 0) cudaSetDevice(prev);
  delete h;
  return from_cuda(e);
}

dms_status dms_cache_reset(dms_cache* h, cudaStream_t stream) {
  const CallRange range("dms_cache_reset");
  if (!h) return DMS_ERR_INVALID;
  if (dms_status s = check_device(h)) return s;
  h->trust_tag = 0;
  note_launch(h, h->device, stream);
  cudaError_t e = cudaMemsetAsync(h->dv.page_table, 0xff, (size_t)h->dv.S * h->dv.mps * sizeof(int32_t), stream);
  if (e == cudaSuccess) e = dms::launch_init_state(h->dv, stream);   // state parity 0 again
  h->launches += 1;
  if (e == cudaSuccess) {
    h->poisoned = false;
    h->par = 0;
  }
  return from_cuda(e);
}

dms_status dms_seq_reset(dms_cache* h, cudaStream_t stream, int32_t seq_id) {
  const CallRange range("dms_seq_reset");
  if (!h || seq_id < 0 || seq_id >= h->cfg.max_seqs) return DMS_ERR_INVALID;
  if (dms_status s = check_usable(h)) return s;
  h->launches += 1;
  h->trust_tag = 0;
  note_launch(h, h->device, stream);
  return from_cuda(dms::launch_reset_seq(h->dv, stream, seq_id));
}

namespace {

// dms_decode_attention's launch, with the stream-list guess of the previous
// attention call on the cache; `early` as recorded for this stream.
cudaError_t attention_impl(dms_cache* h, cudaStream_t stream, bool early, int32_t n_seqs, const int32_t* seq_ids,
                           const void* Q, int32_t num_q_heads, float scale, void* out, dms_dtype out_dtype) {
  const size_t stride = 1 + (size_t)h->cfg.max_seqs;
  const uint64_t k = h->attn_launches;
  const dms::AttnGuess guess{h->attn_guess + ((k + 1) & 1) * stride, h->attn_guess + (k & 1) * stride,
                             early && k > 0};
  const cudaError_t e = dms::launch_attention(h->dv, h->plan, stream, n_seqs, seq_ids, Q, num_q_heads, scale, out,
                                              out_dtype == DMS_F32, counts_for(h, stream), guess);
  if (e == cudaSuccess) h->attn_launches += 1;
  return e;
}

dms_status append_impl(dms_cache* h, cudaStream_t stream, int32_t n_seqs, const int32_t* seq_ids,
                       const int32_t* cu_tokens, int32_t total_tokens, const void* K, const void* V,
                       const uint8_t* alpha, int32_t alpha_channel) {
  const dms::AlphaChoice choice{alpha, alpha_channel, -1};
  if (!h || n_seqs < 0 || n_seqs > h->cfg.max_seqs || total_tokens < 0) return DMS_ERR_INVALID;
  if (dms_status s = check_usable(h)) return s;
  if (alpha_channel >= h->cfg.head_dim) return DMS_ERR_INVALID;
  if (n_seqs == 0) return DMS_OK;
  if (!seq_ids || (total_tokens > 0 && (!K || !V || (alpha_channel < 0 && !alpha)))) return DMS_ERR_INVALID;
  if (!aligned16(K) || !aligned16(V)) return DMS_ERR_INVALID;
  int launches = 0;
  cudaError_t e;
  h->trust_tag = 0;   // the cache changes outside a fused step
  note_launch(h, h->device, stream);
  if (cu_tokens == nullptr) {
    if (total_tokens != n_seqs) return DMS_ERR_INVALID;
    e = dms::launch_append_decode(h->dv, stream, n_seqs, seq_ids, K, V, alpha_src(h, K, nullptr, 0, choice),
                                  &launches);
  } else {
    e = dms::launch_append_bulk(h->dv, stream, n_seqs, seq_ids, cu_tokens, total_tokens, K, V,
                                alpha_src(h, K, nullptr, 0, choice), &launches);
  }
  h->launches += launches;
  return from_cuda(e);
}

dms_status step_impl(dms_cache* h, cudaStream_t stream, int32_t n_seqs, const int32_t* seq_ids, const void* K,
                     const void* V, const dms::AlphaChoice& choice, const void* Q, int32_t num_q_heads,
                     float scale, void* out, dms_dtype out_dtype) {
  if (!h || n_seqs < 0 || n_seqs > h->cfg.max_seqs) return DMS_ERR_INVALID;
  if (dms_status s = check_usable(h)) return s;
  if (num_q_heads < h->cfg.num_kv_heads || num_q_heads % h->cfg.num_kv_heads != 0) return DMS_ERR_INVALID;
  if (num_q_heads / h->cfg.num_kv_heads > dms::kMaxGroup) return DMS_ERR_INVALID;
  if (out_dtype != DMS_BF16 && out_dtype != DMS_F32) return DMS_ERR_INVALID;
  if (choice.channel >= h->cfg.head_dim) return DMS_ERR_INVALID;
  if (choice.channel >= 0 && choice.q_head >= num_q_heads / h->cfg.num_kv_heads) return DMS_ERR_INVALID;
  if (n_seqs == 0) return DMS_OK;
  if (!seq_ids || !K || !V || (choice.channel < 0 && !choice.alpha) || !Q || !out) return DMS_ERR_INVALID;
  if (!aligned16(K) || !aligned16(V) || !aligned16(Q) || !aligned16(out)) return DMS_ERR_INVALID;
  // A fused launch carries host sequence numbers (the state parity it flips,
  // the schedule tags), so a graph replay of it would be wrong: under stream
  // capture the step is issued as the two launches, which read the parity from
  // the device and replay as they were captured.
  const int capture = capturing(stream);
  if (capture < 0) return DMS_ERR_CUDA;
  if (!h->has_step || capture != 0) {
    h->trust_tag = 0;
    note_launch(h, h->device, stream);
    int launches = 0;
    cudaError_t e = dms::launch_append_decode(h->dv, stream, n_seqs, seq_ids, K, V,
                                              alpha_src(h, K, Q, num_q_heads, choice), &launches);
    h->launches += launches;
    if (e != cudaSuccess) return DMS_ERR_CUDA;
    h->launches += 1;
    note_launch(h, h->device, stream);   // the append just before it writes this cache: no early start
    return from_cuda(attention_impl(h, stream, false, n_seqs, seq_ids, Q, num_q_heads, scale, out, out_dtype));
  }
  h->launches += 1;
  const uint64_t tag = ++h->step_tags;   // consecutive with trust_tag whenever that is set
  const bool early = note_launch(h, h->device, stream);
  const cudaError_t e = dms::launch_step(h->dv, h->step_plan, stream, n_seqs, seq_ids, K, V, choice, Q,
                                         num_q_heads, scale, out, out_dtype == DMS_F32, h->par, h->next,
                                         h->trust_tag, tag, early);
  h->trust_tag = e == cudaSuccess ? tag : 0;
  if (e == cudaSuccess) h->par ^= 1;   // the step writes the other copy of the state and flips the parity
  return from_cuda(e);
}

}  // namespace

dms_status dms_append(dms_cache* h, cudaStream_t stream, int32_t n_seqs, const int32_t* seq_ids,
                      const int32_t* cu_tokens, int32_t total_tokens, const void* K, const void* V,
                      const uint8_t* alpha) {
  const CallRange range("dms_append");
  return append_impl(h, stream, n_seqs, seq_ids, cu_tokens, total_tokens, K, V, alpha, -1);
}

dms_status dms_append_keyed(dms_cache* h, cudaStream_t stream, int32_t n_seqs, const int32_t* seq_ids,
                            const int32_t* cu_tokens, int32_t total_tokens, const void* K, const void* V,
                            int32_t alpha_channel) {
  const CallRange range("dms_append_keyed");
  if (alpha_channel < 0) return DMS_ERR_INVALID;
  return append_impl(h, stream, n_seqs, seq_ids, cu_tokens, total_tokens, K, V, nullptr, alpha_channel);
}

dms_status dms_decode_attention(dms_cache* h, cudaStream_t stream, int32_t n_seqs, const int32_t* seq_ids,
                                const void* Q, int32_t num_q_heads, float scale, void* out,
                                dms_dtype out_dtype) {
  const CallRange range("dms_decode_attention");
  if (!h || n_seqs < 0 || n_seqs > h->cfg.max_seqs) return DMS_ERR_INVALID;
  if (dms_status s = check_usable(h)) return s;
  if (num_q_heads < h->cfg.num_kv_heads || num_q_heads % h->cfg.num_kv_heads != 0) return DMS_ERR_INVALID;
  if (num_q_heads / h->cfg.num_kv_heads > dms::kMaxGroup) return DMS_ERR_INVALID;
  if (out_dtype != DMS_BF16 && out_dtype != DMS_F32) return DMS_ERR_INVALID;
  if (n_seqs == 0) return DMS_OK;
  if (!seq_ids || !Q || !out || !aligned16(Q) || !aligned16(out)) return DMS_ERR_INVALID;
  h->launches += 1;
  const bool early = note_launch(h, h->device, stream);
  return from_cuda(attention_impl(h, stream, early, n_seqs, seq_ids, Q, num_q_heads, scale, out, out_dtype));
}

dms_status dms_decode_step(dms_cache* h, cudaStream_t stream, int32_t n_seqs, const int32_t* seq_ids,
                           const void* K, const void* V, const uint8_t* alpha, const void* Q, int32_t num_q_heads,
                           float scale, void* out, dms_dtype out_dtype) {
  const CallRange range("dms_decode_step");
  return step_impl(h, stream, n_seqs, seq_ids, K, V, dms::AlphaChoice{alpha, -1, -1}, Q, num_q_heads, scale, out,
                   out_dtype);
}

dms_status dms_decode_step_keyed(dms_cache* h, cudaStream_t stream, int32_t n_seqs, const int32_t* seq_ids,
                                 const void* K, const void* V, int32_t alpha_channel, const void* Q,
                                 int32_t num_q_heads, float scale, void* out, dms_dtype out_dtype) {
  const CallRange range("dms_decode_step_keyed");
  if (alpha_channel < 0) return DMS_ERR_INVALID;
  return step_impl(h, stream, n_seqs, seq_ids, K, V, dms::AlphaChoice{nullptr, alpha_channel, -1}, Q, num_q_heads,
                   scale, out, out_dtype);
}

dms_status dms_decode_step_qkeyed(dms_cache* h, cudaStream_t stream, int32_t n_seqs, const int32_t* seq_ids,
                                  const void* K, const void* V, const void* Q, int32_t num_q_heads,
                                  int32_t alpha_head, int32_t alpha_channel, float scale, void* out,
                                  dms_dtype out_dtype) {
  const CallRange range("dms_decode_step_qkeyed");
  if (alpha_channel < 0 || alpha_head < 0) return DMS_ERR_INVALID;
  return step_impl(h, stream, n_seqs, seq_ids, K, V, dms::AlphaChoice{nullptr, alpha_channel, alpha_head}, Q,
                   num_q_heads, scale, out, out_dtype);
}

dms_status dms_alpha_from_logit(cudaStream_t stream, const void* X, dms_dtype dtype, int32_t rows,
                                int32_t num_kv_heads, int32_t heads_per_kv, int32_t head, int32_t head_dim,
                                int32_t channel, uint8_t* alpha_out) {
  const CallRange range("dms_alpha_from_logit");
  if (dtype != DMS_BF16 && dtype != DMS_F32) return DMS_ERR_INVALID;
  if (rows < 0 || num_kv_heads < 1 || heads_per_kv < 1 || head < 0 || head >= heads_per_kv) return DMS_ERR_INVALID;
  if (head_dim < 1 || channel < 0 || channel >= head_dim) return DMS_ERR_INVALID;
  if ((int64_t)num_kv_heads * heads_per_kv * head_dim > (int64_t)1 << 30) return DMS_ERR_INVALID;
  if (rows == 0) return DMS_OK;
  if (!X || !alpha_out) return DMS_ERR_INVALID;
  const int eb = dtype == DMS_BF16 ? 2 : 4;
  const dms::AlphaSrc src = dms::alpha_from_queries(X, num_kv_heads, heads_per_kv, head_dim, head, channel, eb);
  return from_cuda(dms::launch_alpha_from_logit(stream, src, rows, alpha_out));
}

dms_status dms_stats(dms_cache* h, cudaStream_t stream, int32_t* retained, int32_t* seen, float* head_cr,
                     int64_t* totals) {
  const CallRange range("dms_stats");
  if (!h) return DMS_ERR_INVALID;
  if (dms_status s = check_usable(h)) return s;
  h->launches += 1;
  // Not recorded: the stats kernel writes no cache state and lets the next
  // kernel start at once (see dms::grid_dependents_launch).
  return from_cuda(dms::launch_stats(h->dv, stream, retained, seen, head_cr, totals));
}

dms_status dms_stats_host(dms_cache* h, cudaStream_t stream, int32_t* retained, int32_t* seen, double* cr_overall) {
  const CallRange range("dms_stats_host");
  if (!h) return DMS_ERR_INVALID;
  if (dms_status s = check_usable(h)) return s;
  const dms::Dev& dv = h->dv;
  const size_t S = dv.S;
  int64_t tot[2] = {0, 0};
  h->launches += 1;
  cudaError_t e = dms::launch_stats(dv, stream, nullptr, nullptr, nullptr, h->totals_dev);
  // The counts of the current state parity: the host's, since the stream's work
  // is ordered and this call syncs it.
  if (e == cudaSuccess && retained)
    e = cudaMemcpyAsync(retained, dv.n + (size_t)h->par * S, S * sizeof(int32_t), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess && seen)
    e = cudaMemcpyAsync(seen, dv.pos + (size_t)h->par * S, S * sizeof(int32_t), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaMemcpyAsync(tot, h->totals_dev, sizeof(tot), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return DMS_ERR_CUDA;
  if (cr_overall) *cr_overall = tot[1] > 0 ? (double)tot[0] / (double)tot[1] : 0.0;
  return DMS_OK;
}

dms_status dms_snapshot(dms_cache* h, cudaStream_t stream, int32_t* page_table, int32_t* n_pages, int32_t* n,
                        int32_t* pos, int32_t* slot_pos, int32_t* free_list, int32_t* free_count) {
  const CallRange range("dms_snapshot");
  if (!h) return DMS_ERR_INVALID;
  if (dms_status s = check_device(h)) return s;
  const dms::Dev& dv = h->dv;
  const size_t S = dv.S;
  cudaError_t e = cudaSuccess;
  auto cp = [&](void* dst, const void* src, size_t bytes) {
    if (dst && e == cudaSuccess) e = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToHost, stream);
  };
  // The current copies of the counts: the stream's work is eager and ordered,
  // so the host's parity is the device's once the copies run.
  cp(page_table, dv.page_table, S * dv.mps * sizeof(int32_t));
  cp(n_pages, dv.n_pages, S * sizeof(int32_t));
  cp(n, dv.n + (size_t)h->par * S, S * sizeof(int32_t));
  cp(pos, dv.pos + (size_t)h->par * S, S * sizeof(int32_t));
  cp(slot_pos, dv.slot_pos, (size_t)dv.max_pages * dms::kPage * sizeof(int32_t));
  cp(free_list, dv.free_list, (size_t)dv.max_pages * sizeof(int32_t));
  cp(free_count, dv.ctrl + dms::kCtrlFree + h->par, sizeof(int32_t));
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  return from_cuda(e);
}

dms_status dms_gather_kv(dms_cache* h, cudaStream_t stream, int32_t seq_id, int32_t kv_head, int32_t rows_cap,
                         void* K_out, void* V_out) {
  const CallRange range("dms_gather_kv");
  if (!h || seq_id < 0 || seq_id >= h->cfg.max_seqs || kv_head < 0 || kv_head >= h->cfg.num_kv_heads)
    return DMS_ERR_INVALID;
  if (dms_status s = check_usable(h)) return s;
  if (rows_cap <= 0) return DMS_OK;
  if (!K_out || !V_out || !aligned16(K_out) || !aligned16(V_out)) return DMS_ERR_INVALID;
  h->launches += 1;
  note_launch(h, h->device, stream);
  return from_cuda(dms::launch_gather(h->dv, stream, seq_id, kv_head, rows_cap, K_out, V_out));
}

dms_status dms_get_status(dms_cache* h, cudaStream_t stream) {
  const CallRange range("dms_get_status");
  if (!h) return DMS_ERR_INVALID;
  if (dms_status s = check_device(h)) return s;
  // The common status word, then the errors the fused steps latched (by parity).
  int32_t words[dms::kCtrlWords] = {};
  cudaError_t e = cudaMemcpyAsync(words, h->dv.ctrl, sizeof(words), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return DMS_ERR_CUDA;
  int32_t word = words[dms::kCtrlStatus];
  if (word == DMS_OK) word = words[dms::kCtrlStepErr];
  if (word == DMS_OK) word = words[dms::kCtrlStepErr + 1];
  if (word != DMS_OK) h->poisoned = true;
  return (dms_status)word;
}

const char* dms_status_string(dms_status s) {
  switch (s) {
    case DMS_OK: return "ok";
    case DMS_ERR_INVALID: return "invalid argument or configuration";
    case DMS_ERR_POOL_EXHAUSTED: return "page pool exhausted";
    case DMS_ERR_CUDA: return "CUDA error";
    case DMS_ERR_TIMEOUT: return "bounded wait timed out inside a kernel";
    case DMS_ERR_POISONED: return "cache poisoned by an earlier device error";
    case DMS_ERR_STREAM_FULL: return "stream page table full";
    case DMS_ERR_BAD_SEQ: return "sequence id out of range";
  }
  return "unknown status";
}

int64_t dms_launch_count(const dms_cache* h) { return h ? h->launches : 0; }

dms_status dms_selftest_bounded_waits(dms_cache* h, cudaStream_t stream, int32_t* timed_out) {
  const CallRange range("dms_selftest_bounded_waits");
  if (!h || !timed_out) return DMS_ERR_INVALID;
  if (dms_status s = check_device(h)) return s;
  h->launches += 1;
  note_launch(h, h->device, stream);   // it writes the cache's status word
  return from_cuda(dms::launch_bounded_wait_selftest(h->dv, stream, timed_out));
}

}  // extern "C"
