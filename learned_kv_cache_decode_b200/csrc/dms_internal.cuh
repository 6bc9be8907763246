// dms_internal.cuh - device state and PTX helpers shared by the libdms kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "dms.h"

namespace dms {

constexpr int kPage = 16;          // tokens per page
constexpr int kMaxGroup = 8;       // query heads per KV head handled by one kernel pass
constexpr int kMaxStreams = 8192;  // max_seqs * num_kv_heads
constexpr int kMaxKvHeads = 256;

// Where the eviction decisions of appended tokens come from: an explicit
// uint8 array [rows][hkv] (channel < 0), or the sign of one designated
// channel of each token's key row: alpha = 1 iff K[row][kvh][channel] > 0
// (the eviction logit read from a repurposed key neuron; zero and NaN keep
// the token).
struct AlphaSrc {
  const uint8_t* alpha;   // [rows][hkv] when channel < 0
  const uint8_t* K;       // [rows][hkv][d] elements
  int channel, hkv, d, elem_bytes;
};

__device__ __forceinline__ int alpha_at(const AlphaSrc& s, size_t row, int kvh) {
  if (s.channel < 0) return s.alpha[row * s.hkv + kvh] != 0;
  const size_t e = (row * s.hkv + kvh) * (size_t)s.d + s.channel;
  const float logit = s.elem_bytes == 2
                          ? __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(s.K)[e] << 16)
                          : reinterpret_cast<const float*>(s.K)[e];
  return logit > 0.f;
}

// Control words (device int32).
enum : int {
  kCtrlStatus = 0,   // latched dms_status, 0 = healthy
  kCtrlFree = 1,     // free-stack depth
  kCtrlPlanned = 2,  // words 2-3: uint64 count of fused-step CTAs done reading the pre-step
                     // state, cumulative over the cache's fused steps (grid per launch)
  kCtrlWords = 8
};

// Everything a kernel needs to know about one cache (device pointers and sizes).
struct Dev {
  int32_t* pos;         // [S] tokens seen
  int32_t* n;           // [S] retained tokens = logical slots in use
  int32_t* n_pages;     // [S]
  int32_t* page_table;  // [S][mps]
  int32_t* ring;        // [S][w] (logical slot << 1) | alpha of the latest token per residue mod w
  int32_t* slot_pos;    // [max_pages * 16] position held by each physical slot
  int32_t* free_list;   // [max_pages] stack, top at ctrl[kCtrlFree] - 1
  int32_t* ctrl;        // [kCtrlWords]
  int32_t* scratch;     // [S] per-call scratch (append bookkeeping)
  uint8_t* kv;          // [max_pages][2][16][d] elements: 16 K rows then 16 V rows per page
  float* part;          // split-K partials [(grid + S)][8][d + 2]
  int32_t* cnt;         // [S] split-K arrival counters
  int S, hkv, d, w, mps, max_pages, max_seqs, elem_bytes;
};

__device__ __forceinline__ void latch(int32_t* ctrl, int code) {
  atomicCAS(&ctrl[kCtrlStatus], 0, code);
}
__device__ __forceinline__ int read_status(const int32_t* ctrl) {
  return *reinterpret_cast<const volatile int32_t*>(&ctrl[kCtrlStatus]);
}

// ---------------------------------------------------------------------------
// Block-wide exclusive scan of one int per thread. `warp_tot` must hold
// blockDim.x / 32 ints of shared memory. Returns the exclusive prefix and
// writes the block total to *total. Contains __syncthreads().
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  int before = 0, all = 0;
  for (int k = 0; k < nw; ++k) {
    int t = warp_tot[k];
    if (k < warp) before += t;
    all += t;
  }
  __syncthreads();
  *total = all;
  return before + x - v;
}

// ---------------------------------------------------------------------------
// PTX wrappers (sm_90+ / sm_100a). Hand-written; no library code.

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// Complete `bytes` of the current phase's expected transactions from a thread.
__device__ __forceinline__ void mbar_complete_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.complete_tx.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait on an mbarrier phase. Gives up after ~2^31 SM cycles (about a
// second), latches DMS_ERR_TIMEOUT and raises the CTA's abort flag. Returns
// false if the data must not be used.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  volatile int* abort_flag, int32_t* ctrl) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > (1ll << 31)) {
      latch(ctrl, DMS_ERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}

// Wait with a time bound only (used to drain copies in flight before exit).
__device__ __forceinline__ void mbar_wait_timed(uint32_t bar, uint32_t parity, int32_t* ctrl) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > (1ll << 31)) {
      latch(ctrl, DMS_ERR_TIMEOUT);
      return;
    }
  }
}

// Spin (one thread) until *flag >= target, bounded by ~2^31 SM cycles; on
// timeout latch DMS_ERR_TIMEOUT and raise the CTA's abort flag. Gives up at
// once when the abort flag is already up. sleep_ns > 0 sleeps between polls.
__device__ __forceinline__ void wait_flag_ge(volatile int* flag, int target, volatile int* abort_flag,
                                             int32_t* ctrl, int sleep_ns = 0) {
  if (*flag >= target) return;
  const long long t0 = clock64();
  while (*flag < target) {
    if (sleep_ns) __nanosleep(sleep_ns);   // leave the issue slots to the warps doing work
    if (*abort_flag) return;
    if (clock64() - t0 > (1ll << 31)) {
      latch(ctrl, DMS_ERR_TIMEOUT);
      *abort_flag = 1;
      return;
    }
  }
}

// TMA tiled load of a 3-D box into shared memory, completing on an mbarrier.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Bring a tensor map into the TMA unit's descriptor cache ahead of its first
// copy (the map is a kernel parameter, readable before any dependency wait).
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Untiled bulk copy global -> shared (size and both addresses 16-B aligned).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// D += A(16x16, row) * B(16x8, col), bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Transpose an 8x8 b16 matrix held in mma fragment layout across the warp.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// Hardware base-2 exponential (MUFU). ex2(-inf) = +0.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

// Device-scope fetch-and-add with acquire-release semantics: the caller's
// earlier writes (and, through a preceding __syncthreads, its CTA's) are
// visible to whoever later acquires the counter, and the caller sees the
// writes released by earlier adders.
__device__ __forceinline__ int atomic_add_acq_rel_gpu(int* p, int v) {
  int old;
  asm volatile("atom.add.acq_rel.gpu.global.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// A global load that stays where it is written, ahead of the asm volatile
// statements that follow it (the TMA copies), instead of being sunk next to
// its first use behind them.
__device__ __forceinline__ int ld_early(const int32_t* p) {
  int v;
  asm volatile("ld.global.cg.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int4 ld_early4(const int4* p) {   // p 16-byte aligned
  int4 v;
  asm volatile("ld.global.cg.v4.s32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}
__device__ __forceinline__ unsigned long long ld_early_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.global.cg.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Programmatic dependent launch. A kernel launched with launch_dependent()
// may start while the previous kernel of its stream is still running; it
// must call grid_dependency_wait() before it touches memory that earlier
// work writes or reads. grid_dependents_launch() lets the next such kernel
// start launching; it never weakens that kernel's own wait.
// Every kernel of this library that writes a cache's state or scratch calls
// grid_dependents_launch() only after its own grid_dependency_wait(), and the
// host records it as the last cache launched on its stream. The stats kernel
// writes neither: it triggers at once and is not recorded. So when a kernel
// starts, every kernel before the last recorded one ahead of it in the stream
// has completed, and that one belongs to the recorded cache. The early starts
// of the attention and fused-step kernels rely on this: they read their
// cache's state before their wait when the record names another cache.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dependents_launch() { asm volatile("griddepcontrol.launch_dependents;"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                    Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Arrive at a named barrier without waiting (the producer side of a
// producer/consumer hand-off; the consumers bar.sync on it). Stores before the
// arrival are visible to the threads that sync on the barrier.
__device__ __forceinline__ void named_barrier_arrive(int id, int threads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Device-scope add with release semantics (no return value): the caller's
// earlier memory operations, and those of its CTA ordered before it by a
// barrier, happen before any acquire that observes the add.
__device__ __forceinline__ void red_add_release_gpu(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Acquire-release fence at device scope (weaker and cheaper than the
// sequentially consistent fence of __threadfence).
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// 64-bit device-scope add with release semantics, no return value.
__device__ __forceinline__ void red_add_release_gpu_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("red.release.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Spin (one thread) until *counter >= target, sleeping between polls, bounded
// like wait_flag_ge.
__device__ __forceinline__ void wait_count_ge(const volatile unsigned long long* counter, unsigned long long target,
                                              volatile int* abort_flag, int32_t* ctrl, int sleep_ns) {
  if (*counter >= target) return;
  const long long t0 = clock64();
  while (*counter < target) {
    __nanosleep(sleep_ns);
    if (*abort_flag) return;
    if (clock64() - t0 > (1ll << 31)) {
      latch(ctrl, DMS_ERR_TIMEOUT);
      *abort_flag = 1;
      return;
    }
  }
}

__device__ __forceinline__ void named_barrier(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ---------------------------------------------------------------------------
// Host-side launchers (defined in dms_append.cu / dms_attention.cu).

cudaError_t prepare_aux_kernels();
cudaError_t launch_init_state(const Dev& dv, cudaStream_t st);
cudaError_t launch_append_decode(const Dev& dv, cudaStream_t st, int n_seqs, const int32_t* seq_ids,
                                 const void* K, const void* V, const uint8_t* alpha, int alpha_channel,
                                 int* launches);
cudaError_t launch_append_bulk(const Dev& dv, cudaStream_t st, int n_seqs, const int32_t* seq_ids,
                               const int32_t* cu_tokens, int total_tokens, const void* K, const void* V,
                               const uint8_t* alpha, int alpha_channel, int* launches);
cudaError_t launch_reset_seq(const Dev& dv, cudaStream_t st, int seq);
cudaError_t launch_bounded_wait_selftest(const Dev& dv, cudaStream_t st, int32_t* timed_out);
cudaError_t launch_stats(const Dev& dv, cudaStream_t st, int32_t* retained, int32_t* seen, float* head_cr,
                         int64_t* totals);
cudaError_t launch_gather(const Dev& dv, cudaStream_t st, int seq, int kvh, int rows_cap, void* Kout,
                          void* Vout);

// Decode attention plan shared by host and launcher.
struct AttnPlan {
  int kernel;        // DMS_ATTN_SIMT or DMS_ATTN_MMA
  int ncw;           // warps per CTA, each with its own TMA page pipeline
  int spw;           // shared-memory stages per warp
  void* fn;          // kernel instantiation
  int grid;          // persistent CTAs
  int threads;
  size_t smem;       // dynamic shared memory bytes
  CUtensorMap tmap;  // pool view for the tiled TMA loads (MMA kernel)
};

cudaError_t attention_prepare(const Dev& dv, int dtype, int kernel_choice, int num_sms, AttnPlan* plan);
// The fused decode step (append + attention in one launch); see dms_decode_step.
cudaError_t step_prepare(const Dev& dv, int dtype, int kernel_choice, int num_sms, AttnPlan* plan);

// The schedule a fused decode step leaves for the next one on the same cache.
// Decode calls the step again and again with the same sequences; the step that
// has just resolved every stream's slots already knows the next step's
// retained counts, positions, leaving slots and page partition, so it writes
// them down and the next step starts its page copies after one round trip
// instead of three (seq ids, then counts, then page ids and window-ring
// entries). The host tags every fused launch (`tag`, never reused) and tells
// the next one which tag to trust: that of the fused step immediately before
// it, or none when another call has changed the cache in between.
//
// Entry i describes call stream i after the step that wrote it.
struct __align__(16) PlanEntry {
  int32_t n, pos;       // retained tokens, tokens seen
  int32_t ring;         // window-ring entry of the token that leaves at the next step
  int32_t seq;          // sequence id of call stream i (stream = seq * hkv + i % hkv)
  unsigned long long tag;
  int32_t first;        // pages of the call streams before stream i (its offset in the range order)
  int32_t pad;
};
// Page list of CTA c for the next step: the physical page ids of its range, in
// range order, with a header of two int4: {tag lo, tag hi, call streams, total
// pages} and {range begin, range end, 0, 0}.
// Double-buffered by tag parity: a step reads the buffer of the tag it trusts
// while it writes the other one.
struct NextPlan {
  PlanEntry* entry;   // [S]
  int4* hdr;          // [2][grid][2]
  int32_t* list;      // [2][grid][cap]
  int cap;            // page ids per CTA: enough for any range of any call (max_pages / grid, rounded up)
};
// `early`: the host knows that the kernel just before this launch in its stream
// does not write this cache, so the step may plan from the schedule and start
// its first page copies before its dependency wait (checked after it).
cudaError_t launch_step(const Dev& dv, const AttnPlan& plan, cudaStream_t st, int n_seqs, const int32_t* seq_ids,
                        const void* K, const void* V, const uint8_t* alpha, int alpha_channel, const void* Q, int hq,
                        float scale, void* out, int out_f32, unsigned long long launch_index,
                        const NextPlan& next, unsigned long long trust_tag, unsigned long long write_tag,
                        bool early);
constexpr int kStepMaxStreams = 1024;   // caches with more streams run the step as two launches

// The stream list of the previous attention call on a cache, kept on the device
// as a guess for the next one: [2][1 + max_seqs] ints, {n_seqs, seq ids...} per
// parity (a launch reads one buffer while it writes the other). `early`: the
// host knows that the kernel just before this launch in its stream does not
// write this cache, so the launch may plan from the guess and the cache state
// and start its first page copies before its dependency wait (checked after it).
struct AttnGuess {
  const int32_t* rd;   // the previous call's list (count < 0: none)
  int32_t* wr;         // this call's list, for the next call
  bool early;
};
cudaError_t launch_attention(const Dev& dv, const AttnPlan& plan, cudaStream_t st, int n_seqs,
                             const int32_t* seq_ids, const void* Q, int hq, float scale, void* out,
                             int out_f32, const AttnGuess& guess);

}  // namespace dms
