// dms_attention.cu - split-K decode attention over the retained pages.
//
// One decode step: for every (sequence, KV head) stream of the call, all g
// query heads of the GQA group attend over the stream's retained tokens,
// which sit densely in logical slots [0, n) of its pages. Decode is bound by
// reading the retained K/V from HBM ("Inference-Time Hyper-Scaling with KV
// Cache Compression", paper summary, Key claims: memory reads dominate
// decode latency at long contexts), so the kernel is built as a page stream:
//
//  * Persistent grid. The call's retained pages, concatenated stream after
//    stream, are cut into equal contiguous ranges, one per CTA (split-K with
//    exact balance whatever the per-stream lengths are). Every CTA derives
//    the plan itself from the retained counts: no host sync, no extra launch.
//  * One producer warp issues TMA copies of whole pages (K rows and V rows
//    are contiguous in a page) into a ring of shared-memory stages guarded by
//    mbarriers; consumer warps take pages round-robin.
//  * Page compute, two variants:
//      MMA  - S^T = K_page (16 x d) * Q^T (d x 8): one m16n8k16 row of tiles
//             per page, the GQA group padded to 8 columns; fp32 online
//             softmax on the fragments; O^T += V^T * P^T with P transposed in
//             registers (movmatrix). The page is loaded through a tensor map
//             with the 128-byte swizzle so ldmatrix reads are conflict-free.
//      SIMT - lanes own head_dim slices; per-token dot products reduced by
//             warp shuffles; online softmax per token. Any dtype.
//  * A piece (stream, page range) of a CTA is merged across its warps in
//    shared memory. A stream split over several CTAs leaves one partial
//    (max, sum, unnormalised output) per CTA; the last CTA to finish the
//    stream (atomic counter) combines them and writes the output. One launch
//    does the whole step.
//  * Tokens past n in a stream's last page are masked by count, not by a
//    mask tensor (the mask is never materialised: paper summary, Key claims,
//    section 3.2 "Performance Considerations").
#include <cstdio>
#include <cstring>
#include <type_traits>

#include "dms_internal.cuh"

namespace dms {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

struct AttnArgs {
  const int32_t* seq_ids;
  const uint8_t* Q;
  uint8_t* out;
  const int32_t* n;
  const int32_t* page_table;
  const uint8_t* kv;
  int32_t* ctrl;
  float* part;
  int32_t* cnt;
  int n_seqs, hkv, g, hq, mps, max_seqs, max_pages, out_f32;
  float sl2e;   // softmax scale * log2(e): scores live in the base-2 domain
};

// Largest i in [0, n] with prefix[i] <= x (prefix is non-decreasing, prefix[0] = 0).
__device__ __forceinline__ int stream_of(const int* prefix, int n, int x) {
  int lo = 0, hi = n;   // invariant: prefix[lo] <= x
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= x) lo = mid; else hi = mid;
  }
  return lo;
}

// CTA that owns global page index x when P pages are cut into G ranges
// [floor(c P / G), floor((c+1) P / G)).
__device__ __forceinline__ int cta_of(long long x, long long P, long long G) {
  return (int)(((x + 1) * G - 1) / P);
}

template <int D>
struct MergeSmem {   // one slot per consumer warp
  float acc[kMaxGroup][D];
  float m[kMaxGroup];
  float l[kMaxGroup];
};

// ---------------------------------------------------------------------------
// MMA page compute (bf16). Lane L holds, for query-head columns
// h0 = 2 (L % 4) and h0 + 1: running max m[2], partial sum l[2] over its own
// tokens, and O^T fragments acc[D/16][4] (rows = head_dim, cols = heads).
template <int D>
struct MmaState {
  uint32_t qb[D / 16][2];   // Q^T B-fragments
  float acc[D / 16][4];
  float m[2], l[2];
};

template <int D>
__device__ __forceinline__ void mma_load_q(MmaState<D>& S, const AttnArgs& a, int b, int kvh, int lane) {
  const int n = lane >> 2;                 // head column of this lane's B fragment
  const bool live = n < a.g;
  const uint32_t* q = reinterpret_cast<const uint32_t*>(
      a.Q + ((size_t)b * a.hq + (size_t)kvh * a.g + (live ? n : 0)) * D * 2);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    S.qb[kk][0] = live ? __ldg(q + kk * 8 + (lane & 3)) : 0u;
    S.qb[kk][1] = live ? __ldg(q + kk * 8 + 4 + (lane & 3)) : 0u;
  }
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
    for (int r = 0; r < 4; ++r) S.acc[mt][r] = 0.f;
  S.m[0] = S.m[1] = -INFINITY;
  S.l[0] = S.l[1] = 0.f;
}

// Address of the 16-byte chunk `chunk` (8 elements of head_dim) of stage row
// `row` (0..15 K, 16..31 V) under the 128-byte TMA swizzle: the page is held
// as D/64 boxes of 32 rows x 128 bytes.
__device__ __forceinline__ uint32_t sw128(uint32_t stage, int row, int chunk) {
  return stage + (uint32_t)((chunk >> 3) * 4096 + row * 128 + (((chunk & 7) ^ (row & 7)) << 4));
}

template <int D>
__device__ __forceinline__ void mma_page(MmaState<D>& S, uint32_t stage, int valid, float sl2e, int lane) {
  // ---- S^T = K * Q^T : rows = 16 tokens, cols = 8 heads
  float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
  const int krow = lane & 15;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t af[4];
    ldsm_x4(sw128(stage, krow, 2 * kk + (lane >> 4)), af);
    if (kk & 1) mma_16816(sb, af, S.qb[kk][0], S.qb[kk][1]);
    else        mma_16816(sa, af, S.qb[kk][0], S.qb[kk][1]);
  }
  float v0 = (sa[0] + sb[0]) * sl2e, v1 = (sa[1] + sb[1]) * sl2e;   // token t0 = lane/4
  float v2 = (sa[2] + sb[2]) * sl2e, v3 = (sa[3] + sb[3]) * sl2e;   // token t0 + 8
  const int t0 = lane >> 2;
  if (valid < kPage) {
    if (t0 >= valid)     { v0 = -INFINITY; v1 = -INFINITY; }
    if (t0 + 8 >= valid) { v2 = -INFINITY; v3 = -INFINITY; }
  }
  // ---- online softmax per head column (tokens spread over lanes with equal lane % 4)
  float mx0 = fmaxf(v0, v2), mx1 = fmaxf(v1, v3);
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
  }
  const float mn0 = fmaxf(S.m[0], mx0), mn1 = fmaxf(S.m[1], mx1);
  const float c0 = ex2(S.m[0] - mn0), c1 = ex2(S.m[1] - mn1);
  const float p0 = ex2(v0 - mn0), p1 = ex2(v1 - mn1);
  const float p2 = ex2(v2 - mn0), p3 = ex2(v3 - mn1);
  S.m[0] = mn0;
  S.m[1] = mn1;
  S.l[0] = S.l[0] * c0 + p0 + p2;
  S.l[1] = S.l[1] * c1 + p1 + p3;
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    S.acc[mt][0] *= c0;
    S.acc[mt][1] *= c1;
    S.acc[mt][2] *= c0;
    S.acc[mt][3] *= c1;
  }
  // ---- P^T as B fragments: transpose the [token][head] C fragments
  const uint32_t pb0 = movmatrix_trans(pack_bf16x2(p0, p1));   // tokens 0..7
  const uint32_t pb1 = movmatrix_trans(pack_bf16x2(p2, p3));   // tokens 8..15
  // ---- O^T += V^T * P^T : rows = head_dim (16 per tile), cols = heads
  const int vrow = 16 + ((lane >> 4) << 3) + (lane & 7);
  const int tk = 2 * (lane & 3);   // tokens of this lane in a0/a1 (and +8 in a2/a3)
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    uint32_t af[4];
    ldsm_x4_trans(sw128(stage, vrow, 2 * mt + ((lane >> 3) & 1)), af);
    if (valid < kPage) {   // rows past n may hold stale bits: zero them
      const uint32_t lo0 = tk < valid ? 0x0000ffffu : 0u, hi0 = tk + 1 < valid ? 0xffff0000u : 0u;
      const uint32_t lo1 = tk + 8 < valid ? 0x0000ffffu : 0u, hi1 = tk + 9 < valid ? 0xffff0000u : 0u;
      af[0] &= lo0 | hi0;
      af[1] &= lo0 | hi0;
      af[2] &= lo1 | hi1;
      af[3] &= lo1 | hi1;
    }
    mma_16816(S.acc[mt], af, pb0, pb1);
  }
}

template <int D>
__device__ __forceinline__ void mma_to_smem(MmaState<D>& S, MergeSmem<D>* slot, int lane) {
  float l0 = S.l[0], l1 = S.l[1];
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  const int h0 = 2 * (lane & 3), r0 = lane >> 2;
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    slot->acc[h0][mt * 16 + r0] = S.acc[mt][0];
    slot->acc[h0 + 1][mt * 16 + r0] = S.acc[mt][1];
    slot->acc[h0][mt * 16 + r0 + 8] = S.acc[mt][2];
    slot->acc[h0 + 1][mt * 16 + r0 + 8] = S.acc[mt][3];
  }
  if (r0 == 0) {
    slot->m[h0] = S.m[0];
    slot->m[h0 + 1] = S.m[1];
    slot->l[h0] = l0;
    slot->l[h0 + 1] = l1;
  }
}

// ---------------------------------------------------------------------------
// SIMT page compute. Lane owns head_dim slice [lane*DPL, lane*DPL + DPL).
template <int D>
struct SimtState {
  static constexpr int DPL = D / 32;
  float q[kMaxGroup][DPL];     // pre-scaled by scale*log2(e)
  float acc[kMaxGroup][DPL];
  float m[kMaxGroup], l[kMaxGroup];   // identical in every lane
};

template <typename E>
__device__ __forceinline__ float to_f32(E x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<uint16_t>(uint16_t x) { return __uint_as_float((uint32_t)x << 16); }

template <int D, typename E>
__device__ __forceinline__ void simt_load_row(const E* row, int lane, float (&x)[D / 32]) {
#pragma unroll
  for (int e = 0; e < D / 32; ++e) x[e] = to_f32<E>(row[lane * (D / 32) + e]);
}

template <int D, typename E>
__device__ __forceinline__ void simt_load_q(SimtState<D>& S, const AttnArgs& a, int b, int kvh, int lane) {
  const E* q = reinterpret_cast<const E*>(a.Q) + ((size_t)b * a.hq + (size_t)kvh * a.g) * D;
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
    float x[D / 32];
    if (h < a.g) simt_load_row<D, E>(q + (size_t)h * D, lane, x);
#pragma unroll
    for (int e = 0; e < D / 32; ++e) {
      S.q[h][e] = h < a.g ? x[e] * a.sl2e : 0.f;
      S.acc[h][e] = 0.f;
    }
    S.m[h] = -INFINITY;
    S.l[h] = 0.f;
  }
}

template <int D, typename E>
__device__ __forceinline__ void simt_page(SimtState<D>& S, const E* stage, int valid, int g, int lane) {
  for (int t = 0; t < valid; ++t) {
    float k[D / 32], v[D / 32];
    simt_load_row<D, E>(stage + (size_t)t * D, lane, k);
    simt_load_row<D, E>(stage + (size_t)(kPage + t) * D, lane, v);
#pragma unroll
    for (int h = 0; h < kMaxGroup; ++h) {
      if (h >= g) break;
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < D / 32; ++e) dot = fmaf(S.q[h][e], k[e], dot);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      const float mn = fmaxf(S.m[h], dot);
      const float c = ex2(S.m[h] - mn), p = ex2(dot - mn);
      S.m[h] = mn;
      S.l[h] = S.l[h] * c + p;
#pragma unroll
      for (int e = 0; e < D / 32; ++e) S.acc[h][e] = fmaf(S.acc[h][e], c, p * v[e]);
    }
  }
}

template <int D>
__device__ __forceinline__ void simt_to_smem(SimtState<D>& S, MergeSmem<D>* slot, int lane) {
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
#pragma unroll
    for (int e = 0; e < D / 32; ++e) slot->acc[h][lane * (D / 32) + e] = S.acc[h][e];
    if (lane == 0) {
      slot->m[h] = S.m[h];
      slot->l[h] = S.l[h];
    }
  }
}

// ---------------------------------------------------------------------------
__device__ __forceinline__ void store_out(const AttnArgs& a, int b, int h, int dd, int D, float v) {
  const size_t idx = ((size_t)b * a.hq + h) * D + dd;
  if (a.out_f32) {
    reinterpret_cast<float*>(a.out)[idx] = v;
  } else {
    uint16_t r;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(v));
    reinterpret_cast<uint16_t*>(a.out)[idx] = r;
  }
}

// Stage ring. Page c of a CTA goes to consumer warp c % NCW, which owns SPW
// private stages and uses them in order: every stage's mbarrier phases are
// then waited on by exactly one warp, one phase after the other, so a
// parity wait can never match a phase two steps old.
template <int NCW, int SPW>
__device__ __forceinline__ int stage_of(int c) { return (c % NCW) * SPW + (c / NCW) % SPW; }
template <int NCW, int SPW>
__device__ __forceinline__ int phase_of(int c) { return (c / NCW) / SPW; }

template <int D, int NCW, int SPW, bool MMA, typename E>
__global__ void __launch_bounds__((NCW + 1) * 32, 1)
attn_kernel(const AttnArgs a, const __grid_constant__ CUtensorMap tmap) {
  constexpr int NSTAGES = NCW * SPW;
  constexpr int kThreads = (NCW + 1) * 32;
  constexpr int kStage = 2 * kPage * D * (int)sizeof(E);   // one page: 16 K rows + 16 V rows
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + NSTAGES * kStage);
  uint64_t* empty = full + NSTAGES;
  int* misc = reinterpret_cast<int*>(empty + NSTAGES);   // [0] abort, [1] ok, [2] last, [3..10] scan
  MergeSmem<D>* mrg = reinterpret_cast<MergeSmem<D>*>(misc + 16);
  int* prefix = reinterpret_cast<int*>(mrg + NCW);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nst = a.n_seqs * a.hkv;
  volatile int* abort_flag = misc;

  if (tid == 0) {
    misc[0] = 0;
    misc[1] = (read_status(a.ctrl) == 0);
    for (int s = 0; s < NSTAGES; ++s) {
      mbar_init(smem_addr(&full[s]), 1);
      mbar_init(smem_addr(&empty[s]), 1);
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (!misc[1]) return;   // poisoned cache: do nothing

  // ---- plan: retained pages per stream of the call, prefix in smem
  {
    const int per = (nst + kThreads - 1) / kThreads;
    const int b0 = min(tid * per, nst), e0 = min(b0 + per, nst);
    int local = 0;
    for (int i = b0; i < e0; ++i) {
      const int seq = a.seq_ids[i / a.hkv];
      int pages = 0;
      if (seq < 0 || seq >= a.max_seqs) {
        latch(a.ctrl, DMS_ERR_BAD_SEQ);
      } else {
        pages = (a.n[seq * a.hkv + i % a.hkv] + kPage - 1) / kPage;
      }
      prefix[i + 1] = pages;
      local += pages;
    }
    int total;
    int run = block_exclusive_scan(local, misc + 3, &total);
    for (int i = b0; i < e0; ++i) {
      run += prefix[i + 1];
      prefix[i + 1] = run;
    }
    if (tid == 0) prefix[0] = 0;
  }
  __syncthreads();
  const long long P = prefix[nst];
  const int G = gridDim.x;

  // Streams with nothing retained produce zeros.
  for (int i = blockIdx.x; i < nst; i += G) {
    if (prefix[i + 1] != prefix[i]) continue;
    const int b = i / a.hkv, kvh = i % a.hkv;
    for (int e = tid; e < a.g * D; e += kThreads) store_out(a, b, kvh * a.g + e / D, e % D, D, 0.f);
  }
  const long long Geff = P < G ? P : G;
  if (blockIdx.x >= Geff) return;
  const int K0 = (int)(blockIdx.x * P / Geff);
  const int K1 = (int)((blockIdx.x + 1) * P / Geff);
  const int ncta = K1 - K0;

  if (warp == NCW) {
    // ================= producer warp =================
    const int bytes_per_row = D * (int)sizeof(E);
    auto lookup = [&](int c) -> int {
      if (c >= ncta) return -1;
      const int kk = K0 + c;
      const int i = stream_of(prefix, nst, kk);
      const int p = kk - prefix[i];
      const int st = a.seq_ids[i / a.hkv] * a.hkv + i % a.hkv;
      int pg = __ldg(a.page_table + (size_t)st * a.mps + p);
      if (pg < 0 || pg >= a.max_pages) {
        latch(a.ctrl, DMS_ERR_INVALID);
        pg = 0;
      }
      return pg;
    };
    int issued = 0;   // lane 0: pages whose copy was issued (in order)
    int pg_next = lookup(lane);
    for (int base = 0; base < ncta; base += 32) {
      const int pg_cur = pg_next;
      pg_next = lookup(base + 32 + lane);   // next batch, overlapped with this one
      const int nb = min(32, ncta - base);
      for (int j = 0; j < nb; ++j) {
        const int pg = __shfl_sync(0xffffffffu, pg_cur, j);
        if (lane == 0 && !*abort_flag) {
          const int c = base + j;
          const int s = stage_of<NCW, SPW>(c), ph = phase_of<NCW, SPW>(c);
          bool go = true;
          if (ph > 0) go = mbar_wait_bounded(smem_addr(&empty[s]), (ph - 1) & 1, abort_flag, a.ctrl);
          if (go) {
            const uint32_t dst = smem_addr(stages + s * kStage);
            const uint32_t bar = smem_addr(&full[s]);
            mbar_arrive_expect_tx(bar, kStage);
            if constexpr (MMA) {
#pragma unroll
              for (int box = 0; box < D / 64; ++box) tma_load_3d(dst + box * 4096, &tmap, bar, box * 64, 0, pg);
            } else {
              bulk_load(dst, a.kv + (size_t)pg * 2 * kPage * bytes_per_row, kStage, bar);
            }
            issued = c + 1;
          }
        }
        __syncwarp();
      }
    }
    // Drain: every issued copy must land before the CTA can exit (bounded).
    // The last NSTAGES issued pages use distinct stages.
    if (lane == 0) {
      for (int c = max(0, issued - NSTAGES); c < issued; ++c)
        mbar_wait_timed(smem_addr(&full[stage_of<NCW, SPW>(c)]), phase_of<NCW, SPW>(c) & 1, a.ctrl);
    }
    return;
  }

  // ================= consumer warps =================
  using State = typename std::conditional<MMA, MmaState<D>, SimtState<D>>::type;
  State S;
  int k = K0;
  while (k < K1) {
    const int i = stream_of(prefix, nst, k);
    const int pstart = prefix[i], pend = prefix[i + 1];
    const int pb = k, pe = min(pend, K1);
    const int b = i / a.hkv, kvh = i % a.hkv;
    const int st = a.seq_ids[b] * a.hkv + kvh;
    const int nn = __ldg(a.n + st);
    const bool whole = (pb == pstart) && (pe == pend);
    if constexpr (MMA) mma_load_q<D>(S, a, b, kvh, lane);
    else simt_load_q<D, E>(S, a, b, kvh, lane);

    const int rel = pb - K0;
    const int c_first = rel + ((warp - rel) % NCW + NCW) % NCW;
    for (int c = c_first; c < pe - K0; c += NCW) {
      const int s = stage_of<NCW, SPW>(c);
      const bool ok = mbar_wait_bounded(smem_addr(&full[s]), phase_of<NCW, SPW>(c) & 1, abort_flag, a.ctrl);
      if (ok) {
        const int p = K0 + c - pstart;
        const int valid = (K0 + c == pend - 1) ? nn - kPage * p : kPage;
        if constexpr (MMA) mma_page<D>(S, smem_addr(stages + s * kStage), valid, a.sl2e, lane);
        else simt_page<D, E>(S, reinterpret_cast<const E*>(stages + s * kStage), valid, a.g, lane);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_addr(&empty[s]));
    }

    // ---- merge the warps' states for this piece
    if constexpr (MMA) mma_to_smem<D>(S, &mrg[warp], lane);
    else simt_to_smem<D>(S, &mrg[warp], lane);
    named_barrier(1, NCW * 32);

    const int slot = blockIdx.x + i;   // partial slot of piece (CTA, stream)
    float* part = a.part + (size_t)slot * kMaxGroup * (D + 2);
    for (int e = tid; e < a.g * D; e += NCW * 32) {
      const int h = e / D, dd = e % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NCW; ++w) M = fmaxf(M, mrg[w].m[h]);
      float L = 0.f, O = 0.f;
#pragma unroll
      for (int w = 0; w < NCW; ++w) {
        const float mw = mrg[w].m[h];
        if (mw == -INFINITY) continue;
        const float sc = ex2(mw - M);
        L += mrg[w].l[h] * sc;
        O += mrg[w].acc[h][dd] * sc;
      }
      if (whole) {
        store_out(a, b, kvh * a.g + h, dd, D, O / L);
      } else {
        part[h * D + dd] = O;
        if (dd == 0) {
          part[kMaxGroup * D + h] = M;
          part[kMaxGroup * D + kMaxGroup + h] = L;
        }
      }
    }
    if (!whole) {
      __threadfence();
      named_barrier(1, NCW * 32);
      const int first = cta_of(pstart, P, Geff), last = cta_of(pend - 1, P, Geff);
      if (tid == 0) misc[2] = (atomicAdd(&a.cnt[i], 1) == last - first);
      named_barrier(1, NCW * 32);
      if (misc[2]) {
        __threadfence();
        for (int e = tid; e < a.g * D; e += NCW * 32) {
          const int h = e / D, dd = e % D;
          float M = -INFINITY;
          for (int c = first; c <= last; ++c)
            M = fmaxf(M, __ldcg(a.part + (size_t)(c + i) * kMaxGroup * (D + 2) + kMaxGroup * D + h));
          float L = 0.f, O = 0.f;
          for (int c = first; c <= last; ++c) {
            const float* pc = a.part + (size_t)(c + i) * kMaxGroup * (D + 2);
            const float sc = ex2(__ldcg(pc + kMaxGroup * D + h) - M);
            L += __ldcg(pc + kMaxGroup * D + kMaxGroup + h) * sc;
            O += __ldcg(pc + h * D + dd) * sc;
          }
          store_out(a, b, kvh * a.g + h, dd, D, O / L);
        }
        if (tid == 0) a.cnt[i] = 0;
      }
    }
    named_barrier(1, NCW * 32);   // merge slots are reused by the next piece
    k = pe;
  }
}

// ---------------------------------------------------------------------------
// Kernel table.

using KernelFn = void (*)(const AttnArgs, const __grid_constant__ CUtensorMap);

struct Variant {
  KernelFn fn;
  int ncw, nstages, stage_bytes, d;
};

constexpr int kNcw = 8;

template <int D, int SPW, bool MMA, typename E>
Variant make_variant() {
  return Variant{attn_kernel<D, kNcw, SPW, MMA, E>, kNcw, kNcw * SPW, 2 * kPage * D * (int)sizeof(E), D};
}

bool pick_variant(int d, int dtype, int kernel, Variant* v) {
  if (kernel == DMS_ATTN_MMA) {
    if (dtype != DMS_BF16) return false;
    *v = d == 64 ? make_variant<64, 2, true, uint16_t>() : make_variant<128, 2, true, uint16_t>();
    return true;
  }
  if (dtype == DMS_BF16)
    *v = d == 64 ? make_variant<64, 2, false, uint16_t>() : make_variant<128, 2, false, uint16_t>();
  else
    *v = d == 64 ? make_variant<64, 2, false, float>() : make_variant<128, 1, false, float>();
  return true;
}

size_t smem_bytes(const Variant& v, int S) {
  const size_t merge = (size_t)v.ncw * (kMaxGroup * (v.d + 2)) * sizeof(float);
  return 1024 + (size_t)v.nstages * v.stage_bytes + 16 * (size_t)v.nstages + 64 + merge +
         (size_t)(S + 1) * sizeof(int);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

}  // namespace

cudaError_t attention_prepare(const Dev& dv, int dtype, int kernel_choice, int num_sms, AttnPlan* plan) {
  int kernel = kernel_choice;
  if (kernel == DMS_ATTN_AUTO) kernel = (dtype == DMS_BF16) ? DMS_ATTN_MMA : DMS_ATTN_SIMT;
  Variant v;
  if (!pick_variant(dv.d, dtype, kernel, &v)) return cudaErrorInvalidValue;
  plan->kernel = kernel;
  plan->threads = (v.ncw + 1) * 32;
  plan->smem = smem_bytes(v, dv.S);
  cudaError_t e = cudaFuncSetAttribute(v.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)plan->smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, v.fn, plan->threads, plan->smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  plan->grid = num_sms * per_sm;

  memset(&plan->tmap, 0, sizeof(plan->tmap));
  if (kernel == DMS_ATTN_MMA) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || fn == nullptr || q != cudaDriverEntryPointSuccess) return cudaErrorNotSupported;
    // Pool viewed as [max_pages][32 rows][d] bf16; box = 64 columns x 32 rows of one page.
    const cuuint64_t dims[3] = {(cuuint64_t)dv.d, 32, (cuuint64_t)dv.max_pages};
    const cuuint64_t strides[2] = {(cuuint64_t)dv.d * 2, (cuuint64_t)dv.d * 2 * 32};
    const cuuint32_t box[3] = {64, 32, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = reinterpret_cast<EncodeTiledFn>(fn)(
        &plan->tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, dv.kv, dims, strides, box, estr,
        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

cudaError_t launch_attention(const Dev& dv, const AttnPlan& plan, cudaStream_t st, int n_seqs,
                             const int32_t* seq_ids, const void* Q, int hq, float scale, void* out,
                             int out_f32) {
  if (n_seqs == 0) return cudaSuccess;
  Variant v;
  pick_variant(dv.d, dv.elem_bytes == 2 ? DMS_BF16 : DMS_F32, plan.kernel, &v);
  AttnArgs a;
  a.seq_ids = seq_ids;
  a.Q = (const uint8_t*)Q;
  a.out = (uint8_t*)out;
  a.n = dv.n;
  a.page_table = dv.page_table;
  a.kv = dv.kv;
  a.ctrl = dv.ctrl;
  a.part = dv.part;
  a.cnt = dv.cnt;
  a.n_seqs = n_seqs;
  a.hkv = dv.hkv;
  a.g = hq / dv.hkv;
  a.hq = hq;
  a.mps = dv.mps;
  a.max_seqs = dv.max_seqs;
  a.max_pages = dv.max_pages;
  a.out_f32 = out_f32;
  a.sl2e = scale * kLog2e;
  v.fn<<<plan.grid, plan.threads, plan.smem, st>>>(a, plan.tmap);
  return cudaGetLastError();
}

}  // namespace dms
