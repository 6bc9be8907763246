// dms_append.cu - cache bookkeeping kernels: decode append, bulk (prefill)
// append, sequence reset, whole-cache reset, statistics, K/V gather.
//
// Retention rule ("Inference-Time Hyper-Scaling with KV Cache Compression",
// paper summary, Key claims and Method, section 3.2): the decision alpha_t
// of a token acts w steps later. With the bound read as "visible iff
// alpha_j == 0 or s - j < w", the token that can leave when token s arrives
// is exactly s - w, so appending s either reuses the slot of s - w (marked)
// or takes a fresh slot. Slots [0, n) therefore stay dense and no validity
// bitmap or mask is ever stored.
#include <algorithm>

#include "dms_internal.cuh"

namespace dms {

namespace {

constexpr int kDecodeThreads = 1024;   // one block per decode append
constexpr int kDecodePre = 4;          // 16-byte K/V vectors held in registers per thread

__device__ __forceinline__ uint8_t* page_row(const Dev& dv, int page, int which, int row, int row_bytes) {
  return dv.kv + ((size_t)page * 2 * kPage + (size_t)which * kPage + row) * row_bytes;
}

// Copy one K or V row (row_bytes, multiple of 16) with a warp of 16-byte vectors.
__device__ __forceinline__ void warp_copy_row(uint8_t* dst, const uint8_t* src, int row_bytes, int lane) {
  const int vec = row_bytes >> 4;
  for (int v = lane; v < vec; v += 32)
    reinterpret_cast<uint4*>(dst)[v] = __ldg(reinterpret_cast<const uint4*>(src) + v);
}

// ---------------------------------------------------------------------------
// Decode append: one token for each stream of the call, in ONE block.
//
// A decode step appends a handful of rows, so the cost of this kernel is
// its chain of dependent memory round trips, each a DRAM latency once the
// attention has flushed L2 with pool reads. One block (no inter-block
// hand-off, no grid-wide counter or fence) keeps the chain at four:
//   1. status, free-stack depth, seq ids, alpha, and the new K/V rows
//      (held in registers when they fit, else prefetched to L2);
//   2. pos and n of every stream;
//   3. the window-ring entry of the token that may leave (s - w);
//   4. the page of the slot (page table), or a popped page for streams
//      that open one (block scan in stream order, so pops are deterministic);
// then the metadata stores and the row copies. Streams beyond the block
// size go in rounds of kDecodeThreads, with the pop ranks carried over.
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__global__ void __launch_bounds__(kDecodeThreads, 1)
append_decode_kernel(Dev dv, int n_seqs, const int32_t* __restrict__ seq_ids,
                     const uint8_t* __restrict__ K, const uint8_t* __restrict__ V, const AlphaSrc asrc) {
  extern __shared__ int s_phys[];   // [nst] physical slot that receives each stream's rows, -1 none
  __shared__ int s_warp[kDecodeThreads / 32];
  constexpr int T = kDecodeThreads;
  const int tid = threadIdx.x;
  const int nst = n_seqs * dv.hkv;
  const int row_bytes = dv.d * dv.elem_bytes;
  const int chunks = row_bytes >> 4;              // 16-byte vectors per row
  const int n_items = nst * 2 * chunks;           // (stream, K or V, vector)

  // Launched early behind the previous kernel of the stream (programmatic
  // dependent launch): nothing is read before this wait.
  grid_dependency_wait();
  grid_dependents_launch();

  // ---- round trip 1 (the free-stack depth of both parities, picked once the
  // parity word is in)
  const int par = read_par(dv.ctrl);
  const int fc0 = read_word(&dv.ctrl[kCtrlFree]), fc1 = read_word(&dv.ctrl[kCtrlFree + 1]);
  auto item_src = [&](int t) -> const uint4* {
    const int i = t / (2 * chunks), which = (t / chunks) & 1, c = t % chunks;
    return reinterpret_cast<const uint4*>((which ? V : K) + (size_t)i * row_bytes) + c;
  };
  uint4 pre[kDecodePre];
#pragma unroll
  for (int p = 0; p < kDecodePre; ++p) {
    const int t = tid + p * T;
    if (t < n_items) pre[p] = __ldg(item_src(t));
  }
  for (int t = kDecodePre * T + tid * 8; t < n_items; t += 8 * T) prefetch_l2(item_src(t));   // 128-B lines
  auto load_ids = [&](int i, int& seq, int& al) {
    seq = -1;
    al = 0;
    if (i < nst) {
      seq = __ldg(seq_ids + i / dv.hkv);
      al = alpha_at(asrc, (size_t)(i / dv.hkv), i % dv.hkv);
    }
  };
  int seq, al;
  load_ids(tid, seq, al);
  if (__syncthreads_or(tid == 0 && read_status(dv.ctrl) != 0)) return;   // poisoned cache
  const Cur cs = cur_state(dv, par);
  const int fc = par ? fc1 : fc0;

  // A call with more streams than threads learns its total page demand
  // first, so that an exhausted pool fails every stream that needs a page.
  int demand = -1;
  if (nst > T) {
    demand = 0;
    for (int r0 = 0; r0 < nst; r0 += T) {
      int sq, a_;
      load_ids(r0 + tid, sq, a_);
      bool need = false;
      if (sq >= 0 && sq < dv.max_seqs) {
        const int st = sq * dv.hkv + (r0 + tid) % dv.hkv;
        const int s = cs.pos[st], nn = cs.n[st];
        const int r = dv.ring[ring_leaving(dv, st, s)];
        need = !((s >= dv.w) && (r & 1)) && (nn % kPage) == 0 && nn / kPage < dv.mps;
      }
      demand += __syncthreads_count(need);
    }
  }

  int popped = 0;   // pages taken by earlier rounds
  int failed = 0;   // pool exhausted
  for (int r0 = 0; r0 < nst; r0 += T) {
    const int i = r0 + tid;
    const bool live = i < nst;
    if (r0 > 0) load_ids(i, seq, al);
    // ---- round trip 2
    const bool good = live && seq >= 0 && seq < dv.max_seqs;
    if (live && !good) latch(dv.ctrl, DMS_ERR_BAD_SEQ);
    const int st = good ? seq * dv.hkv + i % dv.hkv : 0;
    const int s = good ? cs.pos[st] : 0;
    const int nn = good ? cs.n[st] : 0;
    // ---- round trip 3
    const int r = good ? dv.ring[ring_leaving(dv, st, s)] : 0;
    const bool retire = good && (s >= dv.w) && (r & 1);   // token s - w leaves now
    const int slot = retire ? (r >> 1) : nn;
    const int lp = slot / kPage;
    bool go = good;
    bool need = good && !retire && (slot % kPage) == 0;
    if (need && lp >= dv.mps) {
      latch(dv.ctrl, DMS_ERR_STREAM_FULL);
      need = false;
      go = false;
    }
    int total;
    const int rank = block_exclusive_scan(need ? 1 : 0, s_warp, &total);
    const bool fits = !failed && (demand >= 0 ? demand : total) <= fc;
    if (!fits && total > 0) {
      if (tid == 0) latch(dv.ctrl, DMS_ERR_POOL_EXHAUSTED);
      failed = 1;
    }
    if (need && !fits) go = false;   // left unchanged: no stream of this pass pops
    // ---- round trip 4
    int page = -1;
    if (go) {
      if (need) {
        if (in_bounds(fc - 1 - (popped + rank), dv.max_pages, dv.ctrl)) page = dv.free_list[fc - 1 - (popped + rank)];
        else go = false;
      } else {
        page = in_bounds(lp, dv.mps, dv.ctrl) ? dv.page_table[(size_t)st * dv.mps + lp] : -1;
        if (page < 0 || page >= dv.max_pages) {
          latch(dv.ctrl, DMS_ERR_INVALID);
          go = false;
        }
      }
    }
    int phys = -1;
    if (go) {
      if (need) {
        dv.page_table[(size_t)st * dv.mps + lp] = page;
        dv.n_pages[st] = lp + 1;
      }
      if (!retire) cs.n[st] = slot + 1;
      phys = page * kPage + slot % kPage;
      dv.ring[ring_at(dv, st, s)] = (slot << 1) | al;
      cs.pos[st] = s + 1;
      if (in_bounds(phys, (long long)dv.max_pages * kPage, dv.ctrl)) dv.slot_pos[phys] = s;
      else phys = -1;
    }
    if (live) s_phys[i] = phys;
    if (fits) popped += total;
  }
  if (tid == 0 && popped > 0) *cs.free = fc - popped;
  __syncthreads();

  // ---- K and V rows into their slots: 16-byte vectors, consecutive threads
  // on consecutive vectors of a row.
  auto item_dst = [&](int t, int phys) -> uint4* {
    const int which = (t / chunks) & 1, c = t % chunks;
    const int page = phys / kPage, row = phys % kPage;
    return reinterpret_cast<uint4*>(dv.kv + ((size_t)page * 2 * kPage + (size_t)which * kPage + row) * row_bytes) + c;
  };
#pragma unroll
  for (int p = 0; p < kDecodePre; ++p) {
    const int t = tid + p * T;
    if (t < n_items) {
      const int phys = s_phys[t / (2 * chunks)];
      if (phys >= 0) *item_dst(t, phys) = pre[p];
    }
  }
#pragma unroll 4
  for (int t = kDecodePre * T + tid; t < n_items; t += T) {
    const int phys = s_phys[t / (2 * chunks)];
    if (phys >= 0) *item_dst(t, phys) = __ldg(item_src(t));
  }
}

// ---------------------------------------------------------------------------
// Bulk append, pass 1: fresh slots each stream will take -> pages it needs.
// A token j of the call is non-retiring unless j >= w and the token j - w
// (from this call's alpha, or from the window ring for earlier tokens) was
// marked.
__global__ void __launch_bounds__(256)
bulk_count_kernel(Dev dv, int n_seqs, const int32_t* __restrict__ seq_ids,
                  const int32_t* __restrict__ cu, int total_tokens, const AlphaSrc asrc) {
  __shared__ int s_warp[8];
  const int i = blockIdx.x;
  if (read_status(dv.ctrl) != 0) return;
  const int bseq = i / dv.hkv, kvh = i % dv.hkv;
  const int seq = seq_ids[bseq];
  const int t0 = cu[bseq], T = cu[bseq + 1] - t0;
  if (seq < 0 || seq >= dv.max_seqs) {
    if (threadIdx.x == 0) { latch(dv.ctrl, DMS_ERR_BAD_SEQ); dv.scratch[i] = 0; }
    return;
  }
  if (t0 < 0 || T < 0 || t0 + T > total_tokens) {
    if (threadIdx.x == 0) { latch(dv.ctrl, DMS_ERR_INVALID); dv.scratch[i] = 0; }
    return;
  }
  const int st = seq * dv.hkv + kvh;
  const Cur cs = cur_state(dv, read_par(dv.ctrl));
  const int s0 = cs.pos[st];
  int fresh = 0;
  for (int t = threadIdx.x; t < T; t += blockDim.x) {
    const int j = s0 + t;
    int marked = 0;
    if (j >= dv.w) {
      const int jp = j - dv.w;
      marked = (jp >= s0) ? alpha_at(asrc, (size_t)(t0 + jp - s0), kvh)
                          : (dv.ring[ring_at(dv, st, jp)] & 1);
    }
    fresh += !marked;
  }
  int total;
  block_exclusive_scan(fresh, s_warp, &total);
  if (threadIdx.x == 0) {
    const int n_final = cs.n[st] + total;
    const int pages = (n_final + kPage - 1) / kPage;
    if (pages > dv.mps) {
      latch(dv.ctrl, DMS_ERR_STREAM_FULL);
      dv.scratch[i] = 0;
    } else {
      dv.scratch[i] = pages - dv.n_pages[st];
    }
  }
}

// Bulk append, pass 2 (one block): pop the pages in stream order.
__global__ void __launch_bounds__(256)
bulk_pages_kernel(Dev dv, int n_seqs, const int32_t* __restrict__ seq_ids) {
  __shared__ int s_warp[8];
  if (read_status(dv.ctrl) != 0) return;
  const int nst = n_seqs * dv.hkv;
  const int per = (nst + blockDim.x - 1) / blockDim.x;
  const int b = min((int)threadIdx.x * per, nst), e = min(b + per, nst);
  int cnt = 0;
  for (int i = b; i < e; ++i) cnt += dv.scratch[i];
  int total;
  int rank = block_exclusive_scan(cnt, s_warp, &total);
  int32_t* free_depth = cur_state(dv, read_par(dv.ctrl)).free;
  const int fc = *free_depth;
  if (total > fc) {
    if (threadIdx.x == 0) latch(dv.ctrl, DMS_ERR_POOL_EXHAUSTED);
    return;
  }
  for (int i = b; i < e; ++i) {
    const int k = dv.scratch[i];
    if (k == 0) continue;
    const int st = seq_ids[i / dv.hkv] * dv.hkv + i % dv.hkv;
    const int np0 = dv.n_pages[st];
    for (int q = 0; q < k; ++q)
      if (in_bounds(np0 + q, dv.mps, dv.ctrl) && in_bounds(fc - 1 - (rank + q), dv.max_pages, dv.ctrl))
        dv.page_table[(size_t)st * dv.mps + np0 + q] = dv.free_list[fc - 1 - (rank + q)];
    rank += k;
    dv.n_pages[st] = np0 + k;
  }
  __syncthreads();
  if (threadIdx.x == 0) *free_depth = fc - total;
}

// Bulk append, pass 3: slots, window ring, slot tags and rows, one block per
// stream. Tokens go in sub-chunks of at most w consecutive positions, so the
// token j - w every position depends on was settled by an earlier sub-chunk
// (or lives in the ring). Tokens that leave again within this call (marked
// and j + w <= last position) are not copied: their slot is overwritten.
__global__ void __launch_bounds__(256)
bulk_write_kernel(Dev dv, int n_seqs, const int32_t* __restrict__ seq_ids,
                  const int32_t* __restrict__ cu, const uint8_t* __restrict__ K,
                  const uint8_t* __restrict__ V, const AlphaSrc asrc) {
  __shared__ int s_warp[8];
  __shared__ int s_phys[256];
  if (read_status(dv.ctrl) != 0) return;
  const int i = blockIdx.x;
  const int bseq = i / dv.hkv, kvh = i % dv.hkv;
  const int st = seq_ids[bseq] * dv.hkv + kvh;
  const int t0 = cu[bseq], T = cu[bseq + 1] - t0;
  const Cur cs = cur_state(dv, read_par(dv.ctrl));
  const int s0 = cs.pos[st];
  const int s_last = s0 + T - 1;
  const int row_bytes = dv.d * dv.elem_bytes;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
  const int sub = min((int)blockDim.x, dv.w);
  int n_cur = cs.n[st];
  const int32_t* pt = dv.page_table + (size_t)st * dv.mps;

  for (int c0 = 0; c0 < T; c0 += sub) {
    const int t = c0 + tid;
    const bool active = tid < sub && t < T;
    const int j = s0 + t;
    int r = 0;
    bool retire = false;
    if (active) {
      r = dv.ring[ring_leaving(dv, st, j)];   // token j - w (read before the scan's barrier,
      retire = (j >= dv.w) && (r & 1);        // the new entries are written after it)
    }
    int total;
    const int pre = block_exclusive_scan(active && !retire ? 1 : 0, s_warp, &total);
    int phys = -1;
    if (active) {
      const int slot = retire ? (r >> 1) : n_cur + pre;
      const int a = alpha_at(asrc, (size_t)(t0 + t), kvh);
      dv.ring[ring_at(dv, st, j)] = (slot << 1) | a;
      const bool dead = a && (j + dv.w <= s_last);
      const int page = slot / kPage < dv.mps ? pt[slot / kPage] : -1;
      if (page < 0 || page >= dv.max_pages) {
        latch(dv.ctrl, DMS_ERR_INVALID);
      } else if (!dead) {
        phys = page * kPage + slot % kPage;
        dv.slot_pos[phys] = j;   // page checked above: phys < max_pages * 16
      }
    }
    if (tid < 256) s_phys[tid] = phys;
    n_cur += total;
    __syncthreads();
    const int cnt = min(sub, T - c0);
    for (int l = warp; l < cnt; l += nw) {
      const int p = s_phys[l];
      if (p < 0) continue;
      const size_t src = ((size_t)(t0 + c0 + l) * dv.hkv + kvh) * row_bytes;
      warp_copy_row(page_row(dv, p / kPage, 0, p % kPage, row_bytes), K + src, row_bytes, lane);
      warp_copy_row(page_row(dv, p / kPage, 1, p % kPage, row_bytes), V + src, row_bytes, lane);
    }
    __syncthreads();
  }
  if (tid == 0) {
    cs.n[st] = n_cur;
    cs.pos[st] = s0 + T;
  }
}

// ---------------------------------------------------------------------------
// Sequence reset (one block): push pages back, KV head ascending, each
// stream's pages last to first; clear counters and rings.
__global__ void __launch_bounds__(256) reset_seq_kernel(Dev dv, int seq) {
  __shared__ int s_off[kMaxKvHeads + 1];
  __shared__ int s_fc, s_ok;
  const Cur cs = cur_state(dv, read_par(dv.ctrl));
  if (threadIdx.x == 0) {
    s_ok = read_status(dv.ctrl) == 0;
    int acc = 0;
    for (int k = 0; k < dv.hkv; ++k) {
      s_off[k] = acc;
      acc += dv.n_pages[seq * dv.hkv + k];
    }
    s_off[dv.hkv] = acc;
    s_fc = *cs.free;
    if (s_ok && s_fc + acc > dv.max_pages) {
      latch(dv.ctrl, DMS_ERR_INVALID);
      s_ok = 0;
    }
  }
  __syncthreads();
  if (!s_ok) return;
  for (int k = 0; k < dv.hkv; ++k) {
    const int st = seq * dv.hkv + k;
    const int np = s_off[k + 1] - s_off[k];
    for (int p = threadIdx.x; p < np; p += blockDim.x)
      if (in_bounds(s_fc + s_off[k] + (np - 1 - p), dv.max_pages, dv.ctrl) && in_bounds(p, dv.mps, dv.ctrl))
        dv.free_list[s_fc + s_off[k] + (np - 1 - p)] = dv.page_table[(size_t)st * dv.mps + p];
    for (int r = threadIdx.x; r <= dv.w; r += blockDim.x) dv.ring[(size_t)st * (dv.w + 1) + r] = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int k = 0; k < dv.hkv; ++k) {
      const int st = seq * dv.hkv + k;
      cs.n[st] = 0;
      cs.pos[st] = 0;
      dv.n_pages[st] = 0;
    }
    *cs.free = s_fc + s_off[dv.hkv];
  }
}

// Whole-cache reset: fresh free stack (pops 0, 1, 2, ...), empty streams.
__global__ void init_state_kernel(Dev dv) {
  const size_t tid = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
  const size_t nthr = (size_t)gridDim.x * blockDim.x;
  for (size_t k = tid; k < (size_t)dv.max_pages; k += nthr) dv.free_list[k] = dv.max_pages - 1 - (int)k;
  for (size_t k = tid; k < (size_t)dv.S; k += nthr) {
    dv.n_pages[k] = 0;
    dv.scratch[k] = 0;
    dv.cnt[k] = 0;
  }
  for (size_t k = tid; k < 2 * (size_t)dv.S; k += nthr) {   // both parities
    dv.pos[k] = 0;
    dv.n[k] = 0;
  }
  for (size_t k = tid; k < (size_t)dv.S * (dv.w + 1); k += nthr) dv.ring[k] = 0;
  if (tid == 0) {
    for (int k = 0; k < kCtrlWords; ++k) dv.ctrl[k] = 0;   // status, parity 0, no step errors
    dv.ctrl[kCtrlFree] = dv.max_pages;
    dv.ctrl[kCtrlFree + 1] = dv.max_pages;
  }
}

// Statistics (one block).
__global__ void __launch_bounds__(256)
stats_kernel(Dev dv, int32_t* retained, int32_t* seen, float* head_cr, int64_t* totals) {
  // Launched behind the previous kernel of the stream (programmatic dependent
  // launch). It writes no cache state, so the kernel after it may start at
  // once; the host leaves it out of its per-stream record of the last cache
  // launched (see grid_dependents_launch).
  grid_dependents_launch();
  __shared__ unsigned long long s_head[kMaxKvHeads][2];
  for (int h = threadIdx.x; h < dv.hkv; h += blockDim.x) s_head[h][0] = s_head[h][1] = 0;
  grid_dependency_wait();
  const Cur cs = cur_state(dv, read_par(dv.ctrl));
  __syncthreads();
  for (int st = threadIdx.x; st < dv.S; st += blockDim.x) {
    const int r = cs.n[st], p = cs.pos[st];
    if (retained) retained[st] = r;
    if (seen) seen[st] = p;
    atomicAdd(&s_head[st % dv.hkv][0], (unsigned long long)p);
    atomicAdd(&s_head[st % dv.hkv][1], (unsigned long long)r);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long a = 0, b = 0;
    for (int h = 0; h < dv.hkv; ++h) {
      a += s_head[h][0];
      b += s_head[h][1];
      if (head_cr) head_cr[h] = s_head[h][1] ? (float)((double)s_head[h][0] / (double)s_head[h][1]) : 0.f;
    }
    if (totals) {
      totals[0] = (int64_t)a;
      totals[1] = (int64_t)b;
    }
  }
}

// Eviction decisions of `rows` tokens from the sign of a designated logit
// channel: out[row][kvh] = alpha_at(src, row, kvh), one thread per decision.
__global__ void __launch_bounds__(256) alpha_from_logit_kernel(AlphaSrc src, int rows, uint8_t* out) {
  const size_t total = (size_t)rows * src.hkv;
  for (size_t t = blockIdx.x * (size_t)blockDim.x + threadIdx.x; t < total; t += (size_t)gridDim.x * blockDim.x)
    out[t] = (uint8_t)alpha_at(src, t / src.hkv, (int)(t % src.hkv));
}

// Gather the retained rows of one stream in logical slot order (warp per row).
__global__ void __launch_bounds__(256)
gather_kernel(Dev dv, int seq, int kvh, int rows_cap, uint8_t* Kout, uint8_t* Vout) {
  const int st = seq * dv.hkv + kvh;
  const int rows = min(cur_state(dv, read_par(dv.ctrl)).n[st], rows_cap);
  const int row_bytes = dv.d * dv.elem_bytes;
  const int lane = threadIdx.x & 31;
  for (int l = blockIdx.x * 8 + (threadIdx.x >> 5); l < rows; l += gridDim.x * 8) {
    if (!in_bounds(l / kPage, dv.mps, dv.ctrl)) break;
    const int page = dv.page_table[(size_t)st * dv.mps + l / kPage];
    if (page < 0 || page >= dv.max_pages) continue;
    warp_copy_row(Kout + (size_t)l * row_bytes, page_row(dv, page, 0, l % kPage, row_bytes), row_bytes, lane);
    warp_copy_row(Vout + (size_t)l * row_bytes, page_row(dv, page, 1, l % kPage, row_bytes), row_bytes, lane);
  }
}

}  // namespace

// ---------------------------------------------------------------------------

// The attention kernel runs with nearly all of shared memory; giving every
// bookkeeping kernel the same carveout preference spares the SMs a
// reconfiguration between consecutive launches.
cudaError_t prepare_aux_kernels() {
  const void* fns[] = {(const void*)append_decode_kernel, (const void*)bulk_count_kernel,
                       (const void*)bulk_pages_kernel, (const void*)bulk_write_kernel,
                       (const void*)reset_seq_kernel, (const void*)init_state_kernel,
                       (const void*)stats_kernel, (const void*)gather_kernel,
                       (const void*)alpha_from_logit_kernel};
  for (const void* f : fns) {
    cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Failure-detection self-test: the library's two bounded waits, on conditions
// that never come true, in one thread. Each gives up after about 2^31 SM
// cycles, latches DMS_ERR_TIMEOUT and returns; the mbarrier's pending phase is
// then completed by the thread itself, so nothing is left pending at exit.
__global__ void __launch_bounds__(32) bounded_wait_selftest_kernel(int32_t* ctrl, int32_t* timed_out) {
  __shared__ int never;        // a flag nothing sets
  __shared__ int abort_flag;
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  never = 0;
  abort_flag = 0;
  wait_flag_ge(&never, 1, &abort_flag, ctrl);   // raises abort_flag when it gives up
  timed_out[0] = abort_flag != 0;
  abort_flag = 0;
  const uint32_t b = smem_addr(&bar);
  mbar_init(b, 1);
  fence_mbar_init();
  mbar_arrive_expect_tx(b, 16);   // 16 bytes that no copy will bring
  timed_out[1] = mbar_wait_bounded(b, 0, &abort_flag, ctrl) ? 0 : 1;
  mbar_complete_tx(b, 16);        // close the phase
  mbar_wait_timed(b, 0, ctrl);
}

cudaError_t launch_bounded_wait_selftest(const Dev& dv, cudaStream_t st, int32_t* timed_out) {
  bounded_wait_selftest_kernel<<<1, 32, 0, st>>>(dv.ctrl, timed_out);
  return cudaGetLastError();
}

cudaError_t launch_init_state(const Dev& dv, cudaStream_t st) {
  init_state_kernel<<<256, 256, 0, st>>>(dv);
  return cudaGetLastError();
}

cudaError_t launch_append_decode(const Dev& dv, cudaStream_t st, int n_seqs, const int32_t* seq_ids,
                                 const void* K, const void* V, const AlphaSrc& asrc, int* launches) {
  const int nst = n_seqs * dv.hkv;
  if (nst == 0) return cudaSuccess;
  *launches += 1;
  return launch_dependent(append_decode_kernel, dim3(1), dim3(kDecodeThreads), (size_t)nst * sizeof(int), st, dv,
                          n_seqs, seq_ids, (const uint8_t*)K, (const uint8_t*)V, asrc);
}

cudaError_t launch_append_bulk(const Dev& dv, cudaStream_t st, int n_seqs, const int32_t* seq_ids,
                               const int32_t* cu_tokens, int total_tokens, const void* K, const void* V,
                               const AlphaSrc& asrc, int* launches) {
  const int nst = n_seqs * dv.hkv;
  if (nst == 0) return cudaSuccess;
  bulk_count_kernel<<<nst, 256, 0, st>>>(dv, n_seqs, seq_ids, cu_tokens, total_tokens, asrc);
  bulk_pages_kernel<<<1, 256, 0, st>>>(dv, n_seqs, seq_ids);
  bulk_write_kernel<<<nst, 256, 0, st>>>(dv, n_seqs, seq_ids, cu_tokens, (const uint8_t*)K,
                                        (const uint8_t*)V, asrc);
  *launches += 3;
  return cudaGetLastError();
}

cudaError_t launch_reset_seq(const Dev& dv, cudaStream_t st, int seq) {
  reset_seq_kernel<<<1, 256, 0, st>>>(dv, seq);
  return cudaGetLastError();
}

cudaError_t launch_stats(const Dev& dv, cudaStream_t st, int32_t* retained, int32_t* seen, float* head_cr,
                         int64_t* totals) {
  return launch_dependent(stats_kernel, dim3(1), dim3(256), 0, st, dv, retained, seen, head_cr, totals);
}

cudaError_t launch_alpha_from_logit(cudaStream_t st, const AlphaSrc& src, int rows, uint8_t* out) {
  const size_t total = (size_t)rows * src.hkv;
  if (total == 0) return cudaSuccess;
  const int blocks = (int)std::min<size_t>((total + 255) / 256, 4096);
  alpha_from_logit_kernel<<<blocks, 256, 0, st>>>(src, rows, out);
  return cudaGetLastError();
}

cudaError_t launch_gather(const Dev& dv, cudaStream_t st, int seq, int kvh, int rows_cap, void* Kout,
                          void* Vout) {
  const int blocks = max(1, min(1024, (rows_cap + 7) / 8));
  gather_kernel<<<blocks, 256, 0, st>>>(dv, seq, kvh, rows_cap, (uint8_t*)Kout, (uint8_t*)Vout);
  return cudaGetLastError();
}

}  // namespace dms
