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

// What one stream piece costs a CTA of the tensor-core attention kernel, in
// page-times, beyond its pages: the end-of-piece merge (a barrier that waits
// for the warp holding the most pages of the piece, the merge of the warps'
// states, the start of the next piece). The call's pages are cut into CTA
// ranges with each stream weighted by it, so that a range that touches two
// streams gets fewer pages than one inside a stream and both finish together.
// The CUDA-core kernel, bound by arithmetic per page, is cut by pages alone, and
// so is d = 64, whose short pieces measured no better with any weight.
#ifndef DMS_PIECE_COST_D64
#define DMS_PIECE_COST_D64 0
#endif
#ifndef DMS_PIECE_COST_D128
#define DMS_PIECE_COST_D128 20
#endif
__host__ __device__ constexpr int piece_cost(int d, bool mma) {
  return !mma ? 0 : d == 64 ? DMS_PIECE_COST_D64 : DMS_PIECE_COST_D128;
}
constexpr int kMaxPieceCost = DMS_PIECE_COST_D64 > DMS_PIECE_COST_D128 ? DMS_PIECE_COST_D64 : DMS_PIECE_COST_D128;
static_assert(DMS_PIECE_COST_D64 >= 0 && DMS_PIECE_COST_D128 >= 0, "a piece cost is a page count");

// Where the eviction decisions of appended tokens come from: an explicit
// uint8 array [rows][hkv] (channel < 0), or the sign of one designated
// channel of a projection row of each token (the eviction logit read from a
// repurposed neuron; zero and NaN keep the token): alpha = 1 iff
// X[(row * hkv + kvh) * stride + offset] > 0. For the key projection X = K
// [rows][hkv][d], stride = d and offset = channel; for the query projection
// X = Q [rows][hkv * g][d], stride = g * d and offset = head * d + channel,
// `head` being the designated query head within the KV head's group.
struct AlphaSrc {
  const uint8_t* alpha;   // [rows][hkv] when channel < 0
  const uint8_t* X;       // projection rows holding the logit
  int channel;            // < 0: explicit alpha array
  int hkv;
  int stride, offset;     // elements
  int elem_bytes;
};

// alpha from an explicit uint8 array [rows][hkv].
inline AlphaSrc alpha_given(const uint8_t* alpha, int hkv) {
  return AlphaSrc{alpha, nullptr, -1, hkv, 0, 0, 2};
}
// alpha = 1 iff K[row][kvh][channel] > 0.
inline AlphaSrc alpha_from_keys(const void* K, int hkv, int d, int channel, int elem_bytes) {
  return AlphaSrc{nullptr, (const uint8_t*)K, channel, hkv, d, channel, elem_bytes};
}
// alpha = 1 iff Q[row][kvh * g + head][channel] > 0.
inline AlphaSrc alpha_from_queries(const void* Q, int hkv, int g, int d, int head, int channel, int elem_bytes) {
  return AlphaSrc{nullptr, (const uint8_t*)Q, channel, hkv, g * d, head * d + channel, elem_bytes};
}

// logit > 0 decided on the stored bits, so that no flush-to-zero mode can turn a
// positive subnormal into a kept token: the sign bit is clear, the value is not
// +0, and it is at most +inf (larger patterns are NaN).
__device__ __forceinline__ int alpha_at(const AlphaSrc& s, size_t row, int kvh) {
  if (s.channel < 0) return s.alpha[row * s.hkv + kvh] != 0;
  const size_t e = (row * s.hkv + kvh) * (size_t)s.stride + s.offset;
  if (s.elem_bytes == 2) {
    const uint32_t u = reinterpret_cast<const uint16_t*>(s.X)[e];
    return u != 0u && u <= 0x7f80u;
  }
  const uint32_t u = reinterpret_cast<const uint32_t*>(s.X)[e];
  return u != 0u && u <= 0x7f800000u;
}

// Control words (device int32).
//
// The per-stream counts n and pos and the free-stack depth exist twice, and
// the state parity says which copy is current. Every kernel except the fused
// decode step reads and writes the current copy in place. A fused step of
// parity p reads copy p and writes copy 1 - p (every stream: the ones it
// appends to, and a copy of the others), then sets the parity to 1 - p. So no
// CTA of a fused step ever writes a word another CTA of the same launch reads,
// and the step needs no grid-wide wait: its CTAs never wait on one another and
// need not be resident at the same time.
// Errors are latched likewise: the fused step of parity p reads the status
// words kCtrlStatus and kCtrlStepErr + p and latches what its plan finds
// (bad seq id, stream full, pool exhausted) into kCtrlStepErr + 1 - p, which
// no CTA of the launch reads. Every other kernel reads all three words.
enum : int {
  kCtrlStatus = 0,    // latched dms_status, 0 = healthy
  kCtrlFree = 1,      // words 1-2: free-stack depth of each parity
  kCtrlPar = 3,       // state parity (0 or 1)
  kCtrlStepErr = 4,   // words 4-5: errors latched by fused steps, by parity
  kCtrlWords = 8
};

// Everything a kernel needs to know about one cache (device pointers and sizes).
struct Dev {
  int32_t* pos;         // [2][S] tokens seen, one copy per state parity
  int32_t* n;           // [2][S] retained tokens = logical slots in use, per parity
  int32_t* n_pages;     // [S]
  int32_t* page_table;  // [S][mps]
  int32_t* ring;        // [S][w + 1] (logical slot << 1) | alpha of token t at t mod (w + 1)
  int32_t* slot_pos;    // [max_pages * 16] position held by each physical slot
  int32_t* free_list;   // [max_pages] stack, top at the current free-stack depth - 1
  int32_t* ctrl;        // [kCtrlWords]
  int32_t* scratch;     // [S] per-call scratch (append bookkeeping)
  uint8_t* kv;          // [max_pages][2][16][d] elements: 16 K rows then 16 V rows per page
  float* part;          // split-K partials [(grid + S)][8][d + 2]
  int32_t* cnt;         // [S] split-K arrival counters
  int S, hkv, d, w, mps, max_pages, max_seqs, elem_bytes;
  int part_slots;       // partial slots in `part`
};

// Window-ring index of token t: the ring keeps w + 1 entries, so that the entry
// of the token that may leave at step s (s - w) and the entry the new token s
// writes are never the same word.
// (Unsigned arithmetic: no position can give a negative index.)
__device__ __forceinline__ size_t ring_at(const Dev& dv, int stream, int t) {
  return (size_t)stream * (dv.w + 1) + (size_t)((uint32_t)t % (uint32_t)(dv.w + 1));
}
// Entry of the token that leaves when token s arrives, s - w, for s >= w.
__device__ __forceinline__ size_t ring_leaving(const Dev& dv, int stream, int s) {
  return (size_t)stream * (dv.w + 1) + (size_t)(((uint32_t)s + 1u) % (uint32_t)(dv.w + 1));
}

__device__ __forceinline__ void latch(int32_t* ctrl, int code) {
  atomicCAS(&ctrl[kCtrlStatus], 0, code);
}

// Bounds checks of the debug build. A library built with DMS_DEBUG defined
// checks every index the kernels derive by construction (page-table rows and
// columns, partial slots, pool rows, free-stack positions) against its buffer:
// an index out of range latches DMS_ERR_INVALID and the access is skipped,
// never a trap. In the normal build the check compiles to `true`.
#ifdef DMS_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif
__device__ __forceinline__ bool in_bounds(long long idx, long long limit, int32_t* ctrl) {
  if constexpr (kDebugChecks) {
    if (idx < 0 || idx >= limit) {
      latch(ctrl, DMS_ERR_INVALID);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ void latch_word(int32_t* word, int code) { atomicCAS(word, 0, code); }
__device__ __forceinline__ int read_word(const int32_t* p) { return *reinterpret_cast<const volatile int32_t*>(p); }
// Status as every kernel but the fused step sees it: the first error latched anywhere.
__device__ __forceinline__ int read_status(const int32_t* ctrl) {
  const int s = read_word(&ctrl[kCtrlStatus]);
  const int e0 = read_word(&ctrl[kCtrlStepErr]);
  const int e1 = read_word(&ctrl[kCtrlStepErr + 1]);
  return s != 0 ? s : (e0 != 0 ? e0 : e1);
}
__device__ __forceinline__ int read_par(const int32_t* ctrl) { return read_word(&ctrl[kCtrlPar]) & 1; }

// The current copies of the per-stream counts and the free-stack depth.
struct Cur {
  int32_t* n;
  int32_t* pos;
  int32_t* free;
};
__device__ __forceinline__ Cur cur_state(const Dev& dv, int par) {
  return Cur{dv.n + (size_t)par * dv.S, dv.pos + (size_t)par * dv.S, dv.ctrl + kCtrlFree + par};
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

// L2 policy for data read once per launch (the K/V pages): first in line for
// eviction, so that a launch's stream of pages does not push out of L2 what
// is read again (the kernel's code, page tables, schedules, queries, partials).
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// tma_load_3d with an L2 cache policy.
__device__ __forceinline__ void tma_load_3d_hint(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                                 int x, int y, int z, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z), "l"(policy)
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

// bulk_load with an L2 cache policy.
__device__ __forceinline__ void bulk_load_hint(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                               uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
      ::"r"(dst), "l"(src), "r"(bytes), "r"(bar), "l"(policy)
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

__device__ __forceinline__ void named_barrier(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ---------------------------------------------------------------------------
// Host-side launchers (defined in dms_append.cu / dms_attention.cu).

cudaError_t prepare_aux_kernels();
cudaError_t launch_init_state(const Dev& dv, cudaStream_t st);
cudaError_t launch_append_decode(const Dev& dv, cudaStream_t st, int n_seqs, const int32_t* seq_ids,
                                 const void* K, const void* V, const AlphaSrc& asrc, int* launches);
cudaError_t launch_append_bulk(const Dev& dv, cudaStream_t st, int n_seqs, const int32_t* seq_ids,
                               const int32_t* cu_tokens, int total_tokens, const void* K, const void* V,
                               const AlphaSrc& asrc, int* launches);
cudaError_t launch_reset_seq(const Dev& dv, cudaStream_t st, int seq);
cudaError_t launch_bounded_wait_selftest(const Dev& dv, cudaStream_t st, int32_t* timed_out);
cudaError_t launch_stats(const Dev& dv, cudaStream_t st, int32_t* retained, int32_t* seen, float* head_cr,
                         int64_t* totals);
cudaError_t launch_gather(const Dev& dv, cudaStream_t st, int seq, int kvh, int rows_cap, void* Kout,
                          void* Vout);
cudaError_t launch_alpha_from_logit(cudaStream_t st, const AlphaSrc& src, int rows, uint8_t* out);

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
// Entries and lists are double-buffered by tag parity: a step reads the buffers
// of the tag it trusts while it writes the other ones.
struct NextPlan {
  PlanEntry* entry;   // [2][S]
  int4* hdr;          // [2][grid][2]
  int32_t* list;      // [2][grid][cap]
  int cap;            // page ids per CTA: enough for any range of any call
  int S;              // entries per tag parity
};
// Where the eviction decisions of a fused step's new tokens come from: an
// alpha array (channel < 0), or the sign of channel `channel` of the key row
// (q_head < 0) or of query head `q_head` of the KV head's group.
struct AlphaChoice {
  const uint8_t* alpha;
  int channel;
  int q_head;
};
// `par`: the cache's state parity before this step (the host counts the fused
// steps). `early`: the host knows that the kernel just before this launch in
// its stream does not write this cache, so the step may plan from the schedule
// and start its first page copies before its dependency wait (checked after it).
cudaError_t launch_step(const Dev& dv, const AttnPlan& plan, cudaStream_t st, int n_seqs, const int32_t* seq_ids,
                        const void* K, const void* V, const AlphaChoice& alpha, const void* Q, int hq,
                        float scale, void* out, int out_f32, int par, const NextPlan& next,
                        unsigned long long trust_tag, unsigned long long write_tag, bool early);
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
// Retained counts the attention reads: `n` + parity * `stride`, the parity being
// `par` when it is >= 0, else read from the cache's parity word (a launch into a
// stream under capture runs later, after fused steps the host cannot foresee).
// Caller-owned counts: stride 0, par 0.
struct AttnCounts {
  const int32_t* n;
  int stride;
  int par;
};
cudaError_t launch_attention(const Dev& dv, const AttnPlan& plan, cudaStream_t st, int n_seqs,
                             const int32_t* seq_ids, const void* Q, int hq, float scale, void* out,
                             int out_f32, const AttnCounts& counts, const AttnGuess& guess);

}  // namespace dms
