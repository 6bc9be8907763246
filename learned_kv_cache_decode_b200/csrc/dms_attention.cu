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
//    the plan itself on the device: no host sync, no extra launch. A fused
//    step inherits it from the step before (a schedule), and a launch whose
//    previous kernel in the stream belongs to another cache plans and starts
//    its first copies before its dependency wait.
//  * Every warp runs its own page pipeline: it issues TMA copies of whole
//    pages (K rows and V rows are contiguous in a page) into its own ring of
//    shared-memory stages guarded by mbarriers, and computes on them in order.
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
#include <algorithm>
#include <cstdlib>
#include <type_traits>

#include "dms_internal.cuh"

namespace dms {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

constexpr int kRslotUnknown = -2;   // leaving slot not known until the window ring is read

// A decode step fused into the attention launch: the new token of every call
// stream and the cache the append writes.
struct StepArgs {
  const uint8_t* K;       // [n_seqs][hkv][d] new key rows
  const uint8_t* V;       // [n_seqs][hkv][d] new value rows
  AlphaSrc asrc;          // eviction decisions of the new tokens
  Dev dv;                 // the cache, writable
  NextPlan next;          // schedule left by the previous fused step, and the one this step leaves
  unsigned long long trust;   // tag of the schedule to read (0: none, plan from the cache state)
  unsigned long long wtag;    // tag of the schedule this launch writes (trust + 1 when trust != 0)
  int pre;                    // the kernel before this one in the stream does not write this cache
};

struct AttnArgs {
  const int32_t* seq_ids;
  const uint8_t* Q;
  uint8_t* out;
  const int32_t* n;       // retained counts: n + par * n_stride is the current copy
  const int32_t* page_table;
  const uint8_t* kv;
  int32_t* ctrl;
  float* part;
  int32_t* cnt;
  int part_slots;   // partial slots in `part` (debug-build bounds)
  int n_seqs, hkv, g, hq, mps, max_seqs, max_pages, out_f32;
  int n_stride;   // elements between the two parity copies of the counts (0: one copy)
  int par;        // state parity (fused step: before the step); < 0: read the cache's parity word
  float sl2e;   // softmax scale * log2(e): scores live in the base-2 domain
  int spw;      // TMA stages per warp
  int S;        // streams of the cache (sizes the plan arrays in shared memory)
  StepArgs step;   // used by the fused decode-step kernel only
  // Attention alone: the previous call's stream list (a guess for this call's)
  // and the buffer this call leaves its own in; plan before the wait when set.
  const int32_t* guess_rd;
  int32_t* guess_wr;
  int pre_attn;
};

// A retained count as the kernel uses it: clamped to what a stream's page
// table can address, [0, 16 * mps]. Counts the library keeps are always in
// range; caller-owned counts (the allocation-free entry point) are checked here,
// and an out-of-range one latches DMS_ERR_INVALID.
__device__ __forceinline__ int clamp_count(int n, int mps, int32_t* ctrl) {
  const int hi = kPage * mps;
  if (n < 0 || n > hi) {
    latch(ctrl, DMS_ERR_INVALID);
    n = n < 0 ? 0 : hi;
  }
  return n;
}

// Largest i in [0, n] with prefix[i] <= x (prefix is non-decreasing, prefix[0] = 0).
__device__ __forceinline__ int stream_of(const int* prefix, int n, int x) {
  int lo = 0, hi = n;   // invariant: prefix[lo] <= x
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= x) lo = mid; else hi = mid;
  }
  return lo;
}

// Part that holds point x of [0, P) when the line is cut into G parts
// [floor(c P / G), floor((c+1) P / G)), all of them non-empty (G <= P).
__device__ __forceinline__ int range_of(long long x, long long P, long long G) {
  return (int)(((x + 1) * G - 1) / P);
}

// The call's pages cut into CTA ranges, weighted by stream pieces. Page k of
// call stream i sits at cost k + X i on a line of length C = P + X nst: every
// stream adds X page-times, the merge that ends a piece of it, which a CTA
// pays once for each stream its range touches. The line is cut into Geff =
// min(C, G) parts [floor(b C / Geff), floor((b + 1) C / Geff)), none empty,
// and CTA b takes the pages whose cost falls in part b: a contiguous page
// range, empty when the part lies inside the cost of a merge, and CTAs beyond
// Geff hold nothing. The CTAs holding pieces of one stream are consecutive.
// With X = 0 these are the equal page ranges.
struct Cut {
  long long C;
  int Geff, X;
  __device__ __forceinline__ Cut(long long P, int nst, int x, int G) : X(x) {
    C = P + (long long)x * nst;
    Geff = C < G ? (int)C : G;
  }
  // The CTA whose range holds page k of call stream i.
  __device__ __forceinline__ int owner(long long k, int i) const { return range_of(k + (long long)X * i, C, Geff); }
  // First page of CTA b's range, b >= 0 (the end of range b is begin(b + 1)).
  // pf(i): pages of the call streams before stream i, for i in [0, nst].
  template <typename Pf>
  __device__ __forceinline__ long long begin(int b, int nst, Pf pf) const {
    if (b >= Geff) return pf(nst);
    const long long T = (long long)b * C / Geff;   // < C
    int lo = 0, hi = nst;   // the last stream whose cost starts at or before T
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pf(mid) + (long long)X * mid <= T) lo = mid; else hi = mid;
    }
    const long long p0 = pf(lo), into = T - (p0 + (long long)X * lo), n = pf(lo + 1) - p0;
    return p0 + (into < n ? into : n);
  }
};

// Partial result of one (CTA range, stream) piece: unnormalised output
// O[head][d], running max m[head] (base-2 domain) and sum l[head]. The same
// layout serves as a warp's slot in the CTA merge area in shared memory.
template <int D>
struct Partial {
  float O[kMaxGroup][D];
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

// Query of one stream, as this lane's Q^T B-fragments.
template <int D>
struct MmaQuery {
  uint32_t qb[D / 16][2];
};

template <int D>
__device__ __forceinline__ void mma_fetch_q(MmaQuery<D>& Q, const AttnArgs& a, int b, int kvh, int lane) {
  const int n = lane >> 2;                 // head column of this lane's B fragment
  const bool live = n < a.g;
  const uint32_t* q = reinterpret_cast<const uint32_t*>(
      a.Q + ((size_t)b * a.hq + (size_t)kvh * a.g + (live ? n : 0)) * D * 2);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    Q.qb[kk][0] = live ? __ldg(q + kk * 8 + (lane & 3)) : 0u;
    Q.qb[kk][1] = live ? __ldg(q + kk * 8 + 4 + (lane & 3)) : 0u;
  }
}

// Start a piece: take its query, clear the softmax state.
template <int D>
__device__ __forceinline__ void mma_start(MmaState<D>& S, const MmaQuery<D>& Q) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    S.qb[kk][0] = Q.qb[kk][0];
    S.qb[kk][1] = Q.qb[kk][1];
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

// Per-lane byte offsets (within a stage) of the ldmatrix rows this lane
// addresses: K tiles for QK (rows 0..15) and V tiles for PV (rows 16..31).
// Chunk 2t + x and chunk 2t + 8 + x lie at the same place of consecutive
// 64-column boxes (the swizzle sees only the low three chunk bits), so the
// offsets of the first box serve every box: offset(t) = k[t % 4] + (t / 4) * 4096.
template <int D>
struct MmaOffsets {
  static constexpr int kN = D / 16 < 4 ? D / 16 : 4;
  uint32_t k[kN], v[kN];
  __device__ __forceinline__ explicit MmaOffsets(int lane) {
    const int krow = lane & 15;
    const int vrow = 16 + ((lane >> 4) << 3) + (lane & 7);
#pragma unroll
    for (int t = 0; t < kN; ++t) {
      k[t] = sw128(0, krow, 2 * t + (lane >> 4));
      v[t] = sw128(0, vrow, 2 * t + ((lane >> 3) & 1));
    }
  }
  __device__ __forceinline__ uint32_t koff(int t) const { return k[t % kN] + (uint32_t)(t / kN) * 4096u; }
  __device__ __forceinline__ uint32_t voff(int t) const { return v[t % kN] + (uint32_t)(t / kN) * 4096u; }
};

// NP pages of one stream at once: their QK products, one shared online-
// softmax update, then their PV products. Bit r of `rows[p]` says whether
// row r of page p is a token to attend (all 16 except in a stream's last
// page, or where a leaving token's row is masked); the others are
// real (16 except in a stream's last page).
template <int D, int NP>
__device__ __forceinline__ void mma_pages(MmaState<D>& S, const uint32_t (&stage)[NP], const uint32_t (&rows)[NP],
                                          float sl2e, int lane, const MmaOffsets<D>& off) {
  // ---- S^T = K * Q^T per page: rows = 16 tokens, cols = 8 heads
  float v[NP][4];
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t af[4];
      ldsm_x4(stage[p] + off.koff(kk), af);
      if (kk & 1) mma_16816(sb, af, S.qb[kk][0], S.qb[kk][1]);
      else        mma_16816(sa, af, S.qb[kk][0], S.qb[kk][1]);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) v[p][r] = (sa[r] + sb[r]) * sl2e;   // r 0,1: token lane/4; 2,3: +8
  }
  const int t0 = lane >> 2;
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    if (rows[p] != 0xffffu) {
      if (!((rows[p] >> t0) & 1u))       { v[p][0] = -INFINITY; v[p][1] = -INFINITY; }
      if (!((rows[p] >> (t0 + 8)) & 1u)) { v[p][2] = -INFINITY; v[p][3] = -INFINITY; }
    }
  }
  // ---- online softmax per head column (tokens spread over lanes with equal lane % 4)
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    mx0 = fmaxf(mx0, fmaxf(v[p][0], v[p][2]));
    mx1 = fmaxf(mx1, fmaxf(v[p][1], v[p][3]));
  }
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
  }
  const float mn0 = fmaxf(S.m[0], mx0), mn1 = fmaxf(S.m[1], mx1);
  // While every row seen so far is masked the max is -inf; exponents then
  // use 0 as the reference, so that masked rows give 0, not -inf - -inf.
  const float ref0 = mn0 == -INFINITY ? 0.f : mn0, ref1 = mn1 == -INFINITY ? 0.f : mn1;
  float pr[NP][4];
  float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    pr[p][0] = ex2(v[p][0] - ref0);
    pr[p][1] = ex2(v[p][1] - ref1);
    pr[p][2] = ex2(v[p][2] - ref0);
    pr[p][3] = ex2(v[p][3] - ref1);
    sum0 += pr[p][0] + pr[p][2];
    sum1 += pr[p][1] + pr[p][3];
  }
  if (__any_sync(0xffffffffu, (mn0 != S.m[0]) | (mn1 != S.m[1]))) {   // the running max moved
    // a column that has seen nothing (m = -inf) holds l = 0 and O = 0: factor 0
    const float c0 = S.m[0] == -INFINITY ? 0.f : ex2(S.m[0] - mn0);
    const float c1 = S.m[1] == -INFINITY ? 0.f : ex2(S.m[1] - mn1);
    S.l[0] *= c0;
    S.l[1] *= c1;
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      S.acc[mt][0] *= c0;
      S.acc[mt][1] *= c1;
      S.acc[mt][2] *= c0;
      S.acc[mt][3] *= c1;
    }
    S.m[0] = mn0;
    S.m[1] = mn1;
  }
  S.l[0] += sum0;
  S.l[1] += sum1;
  // ---- O^T += V^T * P^T per page: rows = head_dim (16 per tile), cols = heads
  const int tk = 2 * (lane & 3);   // tokens of this lane in a0/a1 (and +8 in a2/a3)
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const uint32_t pb0 = movmatrix_trans(pack_bf16x2(pr[p][0], pr[p][1]));   // tokens 0..7
    const uint32_t pb1 = movmatrix_trans(pack_bf16x2(pr[p][2], pr[p][3]));   // tokens 8..15
    uint32_t keep0 = 0xffffffffu, keep1 = 0xffffffffu;
    if (rows[p] != 0xffffu) {   // masked rows may hold stale bits: zero them
      keep0 = (((rows[p] >> tk) & 1u) ? 0x0000ffffu : 0u) | (((rows[p] >> (tk + 1)) & 1u) ? 0xffff0000u : 0u);
      keep1 = (((rows[p] >> (tk + 8)) & 1u) ? 0x0000ffffu : 0u) | (((rows[p] >> (tk + 9)) & 1u) ? 0xffff0000u : 0u);
    }
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      uint32_t af[4];
      ldsm_x4_trans(stage[p] + off.voff(mt), af);
      af[0] &= keep0;
      af[1] &= keep0;
      af[2] &= keep1;
      af[3] &= keep1;
      mma_16816(S.acc[mt], af, pb0, pb1);
    }
  }
}

// Write a warp's tensor-core state (fragments) into its merge slot.
template <int D>
__device__ __forceinline__ void mma_to_slot(const MmaState<D>& S, Partial<D>* slot, int lane) {
  float l0 = S.l[0], l1 = S.l[1];
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  const int h0 = 2 * (lane & 3), r0 = lane >> 2;
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    slot->O[h0][mt * 16 + r0] = S.acc[mt][0];
    slot->O[h0 + 1][mt * 16 + r0] = S.acc[mt][1];
    slot->O[h0][mt * 16 + r0 + 8] = S.acc[mt][2];
    slot->O[h0 + 1][mt * 16 + r0 + 8] = S.acc[mt][3];
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

// Query of one stream, this lane's head_dim slice of every head, pre-scaled
// by scale * log2(e).
template <int D>
struct SimtQuery {
  float q[kMaxGroup][D / 32];
};

template <int D, typename E>
__device__ __forceinline__ void simt_fetch_q(SimtQuery<D>& Q, const AttnArgs& a, int b, int kvh, int lane) {
  const E* q = reinterpret_cast<const E*>(a.Q) + ((size_t)b * a.hq + (size_t)kvh * a.g) * D;
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
    float x[D / 32];
    if (h < a.g) simt_load_row<D, E>(q + (size_t)h * D, lane, x);
#pragma unroll
    for (int e = 0; e < D / 32; ++e) Q.q[h][e] = h < a.g ? x[e] * a.sl2e : 0.f;
  }
}

template <int D>
__device__ __forceinline__ void simt_start(SimtState<D>& S, const SimtQuery<D>& Q) {
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
#pragma unroll
    for (int e = 0; e < D / 32; ++e) {
      S.q[h][e] = Q.q[h][e];
      S.acc[h][e] = 0.f;
    }
    S.m[h] = -INFINITY;
    S.l[h] = 0.f;
  }
}

template <int D, typename E>
__device__ __forceinline__ void simt_page(SimtState<D>& S, const E* stage, uint32_t rows, int g, int lane) {
  const int end = 32 - __clz(rows);   // one past the highest row to attend
  for (int t = 0; t < end; ++t) {
    if (!((rows >> t) & 1u)) continue;
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
__device__ __forceinline__ void simt_to_slot(const SimtState<D>& S, Partial<D>* slot, int lane) {
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
#pragma unroll
    for (int e = 0; e < D / 32; ++e) slot->O[h][lane * (D / 32) + e] = S.acc[h][e];
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

// Store 4 consecutive output elements (v * inv) of query head h at dims [dd, dd + 4).
__device__ __forceinline__ void store_out4(const AttnArgs& a, int b, int h, int dd, int D, float4 v, float inv) {
  const size_t idx = ((size_t)b * a.hq + h) * D + dd;
  if (a.out_f32) {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + idx) =
        make_float4(v.x * inv, v.y * inv, v.z * inv, v.w * inv);
  } else {
    uint2 r;
    r.x = pack_bf16x2(v.x * inv, v.y * inv);
    r.y = pack_bf16x2(v.z * inv, v.w * inv);
    *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(a.out) + idx) = r;
  }
}

// Online merge of partial (m2, l2, o2) into (m, l, o); scores in base 2. A
// side with m = -inf saw no token and contributes nothing.
__device__ __forceinline__ void merge_into(float& m, float& l, float4& o, float m2, float l2, float4 o2) {
  if (m2 == -INFINITY) return;   // the other side saw nothing
  if (m == -INFINITY) {          // this side saw nothing
    m = m2;
    l = l2;
    o = o2;
    return;
  }
  const float mn = fmaxf(m, m2);
  const float sa = ex2(m - mn), sb = ex2(m2 - mn);   // 0 for a side that saw nothing (m = -inf)
  l = l * sa + l2 * sb;
  o.x = o.x * sa + o2.x * sb;
  o.y = o.y * sa + o2.y * sb;
  o.z = o.z * sa + o2.z * sb;
  o.w = o.w * sa + o2.w * sb;
  m = mn;
}

// Four consecutive elements of a row as floats (p 8-byte aligned for bf16,
// 16-byte aligned for f32).
template <typename E>
__device__ __forceinline__ void load4(const E* p, float (&x)[4]);
template <>
__device__ __forceinline__ void load4<float>(const float* p, float (&x)[4]) {
  const float4 f = *reinterpret_cast<const float4*>(p);
  x[0] = f.x;
  x[1] = f.y;
  x[2] = f.z;
  x[3] = f.w;
}
template <>
__device__ __forceinline__ void load4<uint16_t>(const uint16_t* p, float (&x)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  x[0] = bf16_lo(u.x);
  x[1] = bf16_hi(u.x);
  x[2] = bf16_lo(u.y);
  x[3] = bf16_hi(u.y);
}

// The step's new token of call stream i, for query head h and dims
// [4 d4, 4 d4 + 4): merged into (M, L, O) when `use`. Its score is q . k in
// fp32 from the stored inputs, scaled into base 2 like the page scores.
// Warp-collective: the D/4 lanes of one head reduce the dot product, so
// every lane of the warp calls it, `use` or not.
// The inputs of the new token's term for one merge item: q, k and v at dims
// [4 d4, 4 d4 + 4) of query head h and its stream i.
struct NewTok {
  float q[4], k[4], v[4];
};

template <int D, typename E>
__device__ __forceinline__ void fetch_new_token(const AttnArgs& a, int i, int h, int d4, NewTok& t) {
  const int b = i / a.hkv, kvh = i % a.hkv;
  load4<E>(reinterpret_cast<const E*>(a.Q) + ((size_t)b * a.hq + (size_t)kvh * a.g + h) * D + 4 * d4, t.q);
  load4<E>(reinterpret_cast<const E*>(a.step.K) + (size_t)i * D + 4 * d4, t.k);
  load4<E>(reinterpret_cast<const E*>(a.step.V) + (size_t)i * D + 4 * d4, t.v);
}

// Merge the new token (score q . k in fp32, scaled into base 2 like the page
// scores; value v) into (M, L, O) when `use`. Warp-collective: the D/4 lanes
// of one head reduce the dot product, so every lane of the warp calls it.
template <int D>
__device__ __forceinline__ void apply_new_token(const NewTok& t, float sl2e, bool use, float& M, float& L,
                                                float4& O) {
  float dot = t.q[0] * t.k[0] + t.q[1] * t.k[1] + t.q[2] * t.k[2] + t.q[3] * t.k[3];
#pragma unroll
  for (int o = D / 8; o >= 1; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
  if (use) merge_into(M, L, O, dot * sl2e, 1.f, make_float4(t.v[0], t.v[1], t.v[2], t.v[3]));
}

template <int D, typename E>
__device__ __forceinline__ void add_new_token(const AttnArgs& a, int i, int h, int d4, bool use, float& M,
                                              float& L, float4& O) {
  NewTok t;
  fetch_new_token<D, E>(a, i, h, d4, t);
  apply_new_token<D>(t, a.sl2e, use, M, L, O);
}

// Combine the partials first .. last of stream i into its output, items
// [t_begin, items) with stride t_step (a multiple of 32; every lane of a
// calling warp runs the same iterations). The caller has acquired them.
template <int D, typename E, bool STEP>
__device__ __forceinline__ void combine_stream(const AttnArgs& a, int i, int first, int last, int t_begin,
                                               int t_step, bool add_new) {
  const int b = i / a.hkv, kvh = i % a.hkv;
  const int items = a.g * (D / 4);
  const Partial<D>* base = reinterpret_cast<const Partial<D>*>(a.part) + i;
  if (!in_bounds((long long)last + i, a.part_slots, a.ctrl)) last = first - 1;   // (debug build)
  for (int t0 = 0; t0 < items; t0 += t_step) {
    const int t = t0 + t_begin;
    const bool live = t < items;
    if (!__any_sync(0xffffffffu, live)) break;   // warp-uniform
    const int h = (live ? t : 0) / (D / 4), d4 = (live ? t : 0) % (D / 4);
    NewTok nt;
    if constexpr (STEP) fetch_new_token<D, E>(a, i, h, d4, nt);   // in flight with the partials
    float M = -INFINITY, L = 0.f;
    float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c0 = first; c0 <= last; c0 += 4) {   // loads of 4 pieces in flight at once
      float mc[4], lc[4];
      float4 oc[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + u;
        mc[u] = c <= last ? __ldcg(&base[c].m[h]) : -INFINITY;
        lc[u] = c <= last ? __ldcg(&base[c].l[h]) : 0.f;
        oc[u] = c <= last ? __ldcg(reinterpret_cast<const float4*>(&base[c].O[h][4 * d4]))
                          : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (c0 + u <= last) merge_into(M, L, O, mc[u], lc[u], oc[u]);
    }
    if constexpr (STEP) apply_new_token<D>(nt, a.sl2e, add_new, M, L, O);   // warp-collective
    if (live) store_out4(a, b, kvh * a.g + h, 4 * d4, D, O, L > 0.f ? 1.f / L : 0.f);
  }
}

// The step warp of a fused decode step (one warp per CTA).
//  1. For every call stream, from the pre-step state read by the plan and the
//     leaving slot the consumer warps read from the window ring: does the
//     token at s - w leave now (its slot is reused), or does the new token
//     take the fresh slot n (popping a page when n is a multiple of 16)? Pops
//     are ranked in stream order (warp scan), exactly as dms_append ranks them;
//     a pool too small for all pops fails every stream that needs one.
//  2. Publishes the decisions to the CTA's consumers.
//  3. Writes the state of the next parity that falls to this CTA: the counts of
//     its share of the streams the call does not append to, copied over, and
//     (CTA 0) the parity word and the free-stack depth.
//  4. Writes the outputs of this CTA's streams that had nothing retained (the
//     new token alone: its value row).
//  5. Appends this CTA's call streams (i = blockIdx.x mod gridDim.x):
//     bookkeeping into the next parity and the window ring, and the K/V rows.
// Nothing here waits on another CTA: every word it writes is one that no CTA
// of this launch reads (the other parity's counts, the ring entry of token s
// rather than that of s - w, page-table entries past the pre-step pages, rows
// the attention masks or that lie past the pre-step counts).
template <int D, typename E, int X>
__device__ __forceinline__ void step_warp(const AttnArgs& a, int nst, const int* prefix, const int* sid,
                                       const int* s_nold, const int* s_pos, int* s_rslot, int* s_tslot,
                                       int* s_flag, int* s_rank, int* misc, uint32_t* bits, bool healthy,
                                       volatile int* abort_flag, int K0, int K1) {
  const int lane = threadIdx.x & 31;
  const Dev& dv = a.step.dv;
  const int G = gridDim.x;
  const int par = a.par, nxt = par ^ 1;
  const Cur rd = cur_state(dv, par), wr = cur_state(dv, nxt);
  // Wait (no spinning) until the consumer warps have resolved every stream's
  // leaving slot (s_rslot): they arrive at barrier 2 (waiting there too only
  // when some slot came from the window ring).
  named_barrier(2, blockDim.x);
  if (healthy) {
    const int per = (nst + 31) / 32;   // contiguous streams per lane: the scan keeps stream order
    const int b0 = min(lane * per, nst), e0 = min(b0 + per, nst);
    int cnt = 0;
    for (int i = b0; i < e0; ++i) {
      int f = s_flag[i], ts = -1;
      if (!(f & 4)) {
        const int rs = s_rslot[i];   // token s - w leaves now and s takes its slot
        ts = rs >= 0 ? rs : s_nold[i];
        if (rs < 0 && (ts % kPage) == 0) {
          if (ts / kPage >= dv.mps) {
            f |= 8;
            ts = -1;
          } else {
            f |= 1;
            ++cnt;
          }
        }
      }
      s_tslot[i] = ts;
      s_flag[i] = f;
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    const int fc = misc[12];   // free-stack depth, read by the plan
    const bool fits = total <= fc;
    int rank = incl - cnt;
    for (int i = b0; i < e0; ++i) {
      s_rank[i] = fits ? rank : 0;   // pages popped by the streams before i (a popping stream's rank)
      if (!(s_flag[i] & 1)) continue;
      if (fits) {
        ++rank;
      } else {
        s_tslot[i] = -1;   // pool exhausted: this stream is left unchanged
        s_flag[i] |= 16;
      }
    }
    if (lane == 0) misc[13] = fits ? total : -1;
  }
  __syncwarp();
  if (lane == 0) {
    __threadfence_block();
    *reinterpret_cast<volatile int*>(&misc[15]) = 1;   // the consumers may read the decisions
  }

  // The counts of the next parity. A stream the call appends to is written by
  // the CTA that appends it (below); this CTA copies over its share (stream id
  // = blockIdx.x mod gridDim.x) of the others, or of every stream when the
  // cache is poisoned and nothing is appended.
  const int words = (dv.S + 31) / 32;
  for (int k = lane; k < words; k += 32) bits[k] = 0u;
  __syncwarp();
  if (healthy)
    for (int i = lane; i < nst; i += 32)
      if (!(s_flag[i] & 4)) atomicOr(&bits[sid[i] >> 5], 1u << (sid[i] & 31));
  __syncwarp();
  for (int st = blockIdx.x + G * lane; st < dv.S; st += G * 32) {
    if (healthy && ((bits[st >> 5] >> (st & 31)) & 1u)) continue;
    wr.n[st] = rd.n[st];
    wr.pos[st] = rd.pos[st];
  }
  if (blockIdx.x == 0) {
    // The error of the first call stream that has one (bad seq id before stream
    // full before pool exhausted), found by the whole warp.
    int first = 0x7fffffff;
    if (healthy)
      for (int i = lane; i < nst; i += 32)
        if (s_flag[i] & (4 | 8 | 16)) {
          first = i;
          break;
        }
    first = __reduce_min_sync(0xffffffffu, first);
    if (lane == 0) {
      dv.ctrl[kCtrlPar] = nxt;   // read by the kernels that run after this launch
      if (healthy) {
        if (first < nst) {
          const int f = s_flag[first];
          latch_word(dv.ctrl + kCtrlStepErr + nxt,
                     (f & 4) ? DMS_ERR_BAD_SEQ : (f & 8) ? DMS_ERR_STREAM_FULL : DMS_ERR_POOL_EXHAUSTED);
        }
        *wr.free = misc[13] > 0 ? misc[12] - misc[13] : misc[12];
      } else {
        *wr.free = misc[12];
        latch_word(dv.ctrl + kCtrlStepErr + nxt, misc[16]);   // the error stays visible to the next step
      }
    }
  }
  __syncwarp();
  if (!healthy) return;

  // The streams whose outputs this CTA may produce (whole pieces, and the
  // range's last piece, which it may combine) merge their new token at the
  // end of the piece: pull its query rows and new K and V rows into L2 while
  // the pages stream, one prefetch per 128-byte line.
  for (int k = K0; k < K1;) {
    const int i = stream_of(prefix, nst, k);
    const int pe = min(prefix[i + 1], K1);
    if (prefix[i] >= K0 || pe == K1) {
      const int b = i / a.hkv, kvh = i % a.hkv;
      const int qlines = a.g * D * (int)sizeof(E) / 128, rlines = D * (int)sizeof(E) / 128;
      const uint8_t* qrow = a.Q + ((size_t)b * a.hq + (size_t)kvh * a.g) * D * sizeof(E);
      const uint8_t* krow = a.step.K + (size_t)i * D * sizeof(E);
      const uint8_t* vrow = a.step.V + (size_t)i * D * sizeof(E);
      for (int l = lane; l < qlines + 2 * rlines; l += 32) {
        const uint8_t* p = l < qlines ? qrow + (size_t)l * 128
                                      : (l < qlines + rlines ? krow + (size_t)(l - qlines) * 128
                                                             : vrow + (size_t)(l - qlines - rlines) * 128);
        asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
      }
    }
    k = pe;
  }

  // Streams with nothing retained before the step attend to the new token alone.
  for (int i = blockIdx.x; i < nst; i += G) {
    if (prefix[i + 1] != prefix[i]) continue;
    const int b = i / a.hkv, kvh = i % a.hkv;
    const bool app = s_tslot[i] >= 0;
    for (int e = lane; e < a.g * (D / 4); e += 32) {
      const int h = e / (D / 4), d4 = e % (D / 4);
      float v4[4] = {0.f, 0.f, 0.f, 0.f};
      if (app) load4<E>(reinterpret_cast<const E*>(a.step.V) + (size_t)i * D + 4 * d4, v4);
      store_out4(a, b, kvh * a.g + h, 4 * d4, D, make_float4(v4[0], v4[1], v4[2], v4[3]), 1.f);
    }
  }

  // This CTA's page list for the next step on the same streams. After this
  // step, stream i holds its old pages plus the one it popped, so its pages
  // start at prefix[i] + s_rank[i] in the call's concatenated order, and the
  // next step cuts P + pops pages into the same kind of ranges. Existing pages
  // come from the page table (this step writes only entries past them), a
  // popped one from the free stack (never written by a step). Nothing reads
  // this buffer during this launch: it is the one of the other tag parity.
  // Eight loads per lane are in flight at a time; the first batch's loads go
  // out together with those of the appends below.
  const int wbuf = (int)(a.step.wtag & 1ull);
  long long c0 = 0, c1 = 0;
  int32_t* lst = nullptr;
  size_t cell = 0;
  if (a.step.next.entry != nullptr && misc[13] >= 0) {
    const long long P2 = (long long)prefix[nst] + misc[13];
    const Cut cut2(P2, nst, X, G);
    auto pf2 = [&](int i) -> long long { return i < nst ? (long long)prefix[i] + s_rank[i] : P2; };
    c0 = cut2.begin(blockIdx.x, nst, pf2);
    c1 = cut2.begin(blockIdx.x + 1, nst, pf2);
    if (c1 - c0 <= a.step.next.cap) {
      cell = (size_t)wbuf * G + blockIdx.x;
      lst = a.step.next.list + cell * a.step.next.cap;
      if (lane == 0) {
        a.step.next.hdr[2 * cell] = make_int4((int)(uint32_t)a.step.wtag, (int)(uint32_t)(a.step.wtag >> 32), nst, (int)P2);
        a.step.next.hdr[2 * cell + 1] = make_int4((int)c0, (int)c1, 0, 0);
      }
    }
  }
  const int fc = misc[12];
  // Page id of position kk of the next step's concatenated order (kk < c1).
  auto list_page = [&](long long kk) -> int {
    int lo = 0, hi = nst;   // largest i with prefix[i] + s_rank[i] <= kk
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (prefix[mid] + s_rank[mid] <= kk) lo = mid; else hi = mid;
    }
    const int p = (int)(kk - prefix[lo] - s_rank[lo]);
    if (p < prefix[lo + 1] - prefix[lo]) {
      if (in_bounds(sid[lo], dv.S, a.ctrl) && in_bounds(p, dv.mps, a.ctrl))
        return __ldg(dv.page_table + (size_t)sid[lo] * dv.mps + p);
    } else if (in_bounds(fc - 1 - s_rank[lo], dv.max_pages, a.ctrl)) {
      return __ldg(dv.free_list + (fc - 1 - s_rank[lo]));
    }
    return 0;
  };
  int lv0 = 0, lv1 = 0, lv2 = 0, lv3 = 0, lv4 = 0, lv5 = 0, lv6 = 0, lv7 = 0;   // first batch, in registers
  if (lst != nullptr) {
    if (c0 + lane < c1) lv0 = list_page(c0 + lane);
    if (c0 + lane + 32 < c1) lv1 = list_page(c0 + lane + 32);
    if (c0 + lane + 64 < c1) lv2 = list_page(c0 + lane + 64);
    if (c0 + lane + 96 < c1) lv3 = list_page(c0 + lane + 96);
    if (c0 + lane + 128 < c1) lv4 = list_page(c0 + lane + 128);
    if (c0 + lane + 160 < c1) lv5 = list_page(c0 + lane + 160);
    if (c0 + lane + 192 < c1) lv6 = list_page(c0 + lane + 192);
    if (c0 + lane + 224 < c1) lv7 = list_page(c0 + lane + 224);
  }

  // Append this CTA's call streams: bookkeeping into the next parity and the
  // window ring (the entry of token s, never the one of s - w that the plan
  // reads), the K/V rows into a masked row or one past the pre-step count. A
  // stream left unchanged (stream full, pool exhausted) carries its counts over.
  // Every load of one stream's append (its page id, the ring entry for the next
  // step's schedule, the new K and V rows) is issued before any store: one
  // memory round trip per stream, which the page stream of the consumers keeps
  // long.
  constexpr int kRowBytes = D * (int)sizeof(E);
  constexpr int kVec = kRowBytes / 16;                  // 16-byte vectors per row
  constexpr int kPerLane = (2 * kVec + 31) / 32;        // K and V vectors per lane
  PlanEntry* entries = a.step.next.entry != nullptr ? a.step.next.entry + (size_t)wbuf * a.step.next.S : nullptr;
  for (int i = blockIdx.x; i < nst; i += G) {
    const int ts = s_tslot[i];
    const int st = sid[i], s = s_pos[i], f = s_flag[i];
    if (f & 4) continue;   // bad seq id: no stream
    int page = -1, rn = 0;
    uint4 x[kPerLane];
    if (ts >= 0) {
      if (lane == 0) {
        if (f & 1) {
          if (in_bounds(fc - 1 - s_rank[i], dv.max_pages, a.ctrl)) page = dv.free_list[fc - 1 - s_rank[i]];
        } else if (in_bounds(st, dv.S, a.ctrl) && in_bounds(ts / kPage, dv.mps, a.ctrl)) {
          page = dv.page_table[(size_t)st * dv.mps + ts / kPage];
        }
      }
      if (lane == 1 && entries != nullptr && dv.w > 1) rn = dv.ring[ring_leaving(dv, st, s + 1)];
#pragma unroll
      for (int c = 0; c < kPerLane; ++c) {
        const int v = lane + 32 * c;
        if (v < 2 * kVec)
          x[c] = __ldg(reinterpret_cast<const uint4*>((v >= kVec ? a.step.V : a.step.K) + (size_t)i * kRowBytes) +
                       (v % kVec));
      }
    }
    page = __shfl_sync(0xffffffffu, page, 0);
    rn = __shfl_sync(0xffffffffu, rn, 1);
    if (page < 0 || page >= dv.max_pages) {
      if (lane == 0) {
        if (ts >= 0) latch(a.ctrl, DMS_ERR_INVALID);
        wr.n[st] = s_nold[i];
        wr.pos[st] = s;
      }
      continue;
    }
    if (lane == 0) {
      const int lp = ts / kPage;
      const int nnew = s_rslot[i] < 0 ? s_nold[i] + 1 : s_nold[i];
      const int rent = (ts << 1) | ((f >> 1) & 1);
      if ((f & 1) && in_bounds(lp, dv.mps, a.ctrl)) {
        dv.page_table[(size_t)st * dv.mps + lp] = page;
        dv.n_pages[st] = lp + 1;
      }
      wr.n[st] = nnew;
      wr.pos[st] = s + 1;
      dv.ring[ring_at(dv, st, s)] = rent;
      dv.slot_pos[(size_t)page * kPage + ts % kPage] = s;
      if (entries != nullptr) {
        // The schedule entry of call stream i for the next step: the ring entry
        // of the token that leaves then (s + 1 - w), the one just written when
        // w = 1, else one this step leaves alone.
        PlanEntry* e = entries + i;
        *reinterpret_cast<int4*>(e) = make_int4(nnew, s + 1, dv.w == 1 ? rent : rn, st / a.hkv);
        e->tag = a.step.wtag;
        e->first = prefix[i] + s_rank[i];
      }
    }
#pragma unroll
    for (int c = 0; c < kPerLane; ++c) {
      const int v = lane + 32 * c;
      if (v < 2 * kVec) {
        const int which = v >= kVec;
        reinterpret_cast<uint4*>(dv.kv + ((size_t)page * 2 * kPage + (size_t)which * kPage + ts % kPage) * kRowBytes)
            [v % kVec] = x[c];
      }
    }
  }

  if (lst != nullptr) {
    const long long l0 = lane;
    if (c0 + l0 < c1) lst[l0] = lv0;
    if (c0 + l0 + 32 < c1) lst[l0 + 32] = lv1;
    if (c0 + l0 + 64 < c1) lst[l0 + 64] = lv2;
    if (c0 + l0 + 96 < c1) lst[l0 + 96] = lv3;
    if (c0 + l0 + 128 < c1) lst[l0 + 128] = lv4;
    if (c0 + l0 + 160 < c1) lst[l0 + 160] = lv5;
    if (c0 + l0 + 192 < c1) lst[l0 + 192] = lv6;
    if (c0 + l0 + 224 < c1) lst[l0 + 224] = lv7;
    for (long long base = c0 + 32 * 8; base < c1; base += 32 * 8) {   // longer ranges: 8 loads in flight per lane
      int v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = base + lane + 32 * u < c1 ? list_page(base + lane + 32 * u) : 0;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (base + lane + 32 * u < c1) lst[base + lane + 32 * u - c0] = v[u];
    }
  }

  // The stream of the range's last piece, when other CTAs hold pieces of it:
  // if they have all published theirs by the time the consumers start that
  // piece (they usually are: the next CTA finishes the stream's tail at the
  // start of its range), the consumers will be the last to finish the stream
  // and can combine without publishing their own piece and taking a ticket.
  // The acquire read makes the other pieces' partials visible to them (CTA
  // fence, then the flag). The wait for the consumers is bounded; giving up
  // only skips the shortcut.
  if (lane == 0 && K1 > K0) {
    const int il = stream_of(prefix, nst, K1 - 1);
    if (prefix[il] < K0 || prefix[il + 1] > K1) {
      const long long t0 = clock64();
      bool started = true;
      while (*reinterpret_cast<volatile int*>(&misc[17]) == 0) {
        __nanosleep(256);
        if (*abort_flag || clock64() - t0 > (1ll << 31)) {
          started = false;
          break;
        }
      }
      if (started) {
        const Cut cut(prefix[nst], nst, X, G);
        const int first = cut.owner(prefix[il], il), last = cut.owner(prefix[il + 1] - 1, il);
        const bool done = ld_acquire_gpu(&a.cnt[il]) == last - first;
        __threadfence_block();
        *reinterpret_cast<volatile int*>(&misc[3]) = done ? 1 : 2;
      }
    }
  }
}

// One page (16 K rows, then 16 V rows) into a warp's stage j % spw, completing
// on that stage's mbarrier. Called by one lane.
template <int D, bool MMA, typename E>
__device__ __forceinline__ void issue_page(uint64_t* myfull, uint8_t* mystage, int spw, int j, int pg,
                                           const CUtensorMap* tmap, const uint8_t* kv) {
  constexpr int kStage = 2 * kPage * D * (int)sizeof(E);
  const int s = j % spw;
  const uint32_t bar = smem_addr(&myfull[s]);
  const uint32_t dst = smem_addr(mystage + (size_t)s * kStage);
  mbar_arrive_expect_tx(bar, kStage);
  if constexpr (MMA) {
#pragma unroll
    const uint64_t pol = l2_evict_first();   // pages are read once per launch
    for (int box = 0; box < D / 64; ++box) tma_load_3d_hint(dst + box * 4096, tmap, bar, box * 64, 0, pg, pol);
  } else {
    bulk_load_hint(dst, kv + (size_t)pg * kStage, kStage, bar, l2_evict_first());
  }
}

// Shared-memory layout of one CTA (byte offsets from a 1024-aligned base).
struct SmemLayout {
  int stages, bars, misc, merge, prefix, sid, step, bits, total;
};

__host__ __device__ inline SmemLayout smem_layout(int ncw, int spw, int stage_bytes, int d, int S, bool step) {
  SmemLayout L;
  L.stages = 0;
  L.bars = ncw * spw * stage_bytes;
  L.misc = L.bars + 8 * ncw * spw;
  L.merge = L.misc + 128;
  L.prefix = L.merge + ncw * kMaxGroup * (d + 2) * 4;
  L.sid = L.prefix + (S + 1) * 4;
  L.step = L.sid + S * 4;
  L.bits = L.step + (step ? 6 * S * 4 : 0);               // per-stream step decisions
  L.total = L.bits + (step ? ((S + 31) / 32) * 4 : 0);   // the call's streams, one bit per cache stream
  return L;
}

// Split-K over CTA ranges. The call's retained pages, stream after stream,
// are cut into gridDim.x contiguous ranges, one per CTA, of equal cost (pages,
// plus a fixed cost for each stream piece: see Cut). Page c of a
// range goes to warp c % NCW, which runs its own TMA pipeline over `spw`
// private stages: it refills a stage as soon as it has computed on it, and
// every stage's mbarrier phases are waited on by that one warp, in order.
// At the end of each stream piece the warps' softmax states are merged in
// shared memory; a split stream leaves one partial per CTA and the last CTA
// to finish it combines them (a few partials per stream). The next piece's
// query is loaded before the merge, and the copies already in flight keep
// HBM busy while the CTA merges.
//
// STEP: the launch also appends this step's token of every stream (the
// decode step fused into one launch). The attention runs over the cache as
// it was before the step: the row of the token that leaves at this step is
// masked, and the new token enters every stream's final merge from its input
// row. A ninth warp resolves each stream's slots (window ring, page pops in
// stream order, the same rule as dms_append) and writes the append:
// bookkeeping into the other state parity and the K/V rows. A row it
// overwrites is a masked one or lies past the pre-step count, so no CTA ever
// attends a row being written, and no CTA waits for another.
template <int D, int NCW, int NB, bool MMA, typename E, bool STEP>
__global__ void __launch_bounds__((NCW + (STEP ? 1 : 0)) * 32, 1)
attn_kernel(const AttnArgs a, const __grid_constant__ CUtensorMap tmap) {
  constexpr int kThreads = (NCW + (STEP ? 1 : 0)) * 32;   // consumers (+ the step warp)
  constexpr int kMergeThreads = NCW * 32;                  // the consumer warps
  constexpr int kStage = 2 * kPage * D * (int)sizeof(E);   // one page: 16 K rows + 16 V rows
  constexpr int kX = piece_cost(D, MMA);                   // weight of a stream piece in the cut
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The 128-byte TMA swizzle needs 1024-aligned stages. The declaration asks
  // for that alignment and the launch reserves no slack for rounding up, so a
  // base that is not aligned would overrun: the CTA then reports and stops
  // before touching shared memory (uniform over the CTA).
  uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  const int spw = a.spw;
  const SmemLayout lay = smem_layout(NCW, spw, kStage, D, a.S, STEP);
  {
    uint32_t dyn;
    asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn));
    if ((uint32_t)(smem - smem_raw) + (uint32_t)lay.total > dyn) {
      if (threadIdx.x == 0) latch(a.ctrl, DMS_ERR_INVALID);
      return;
    }
  }
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.bars);
  // misc: [0] abort, [1] ok, [2] last flag, [3 .. 3+warps) scan scratch (after the plan, STEP:
  // [3] the other pieces of the range's last stream are all published (1) or not (2), [4] the
  // consumers' snapshot of [3]), [12] free-stack depth
  // and [13] pages popped by this step (-1: pool exhausted), [14] stream whose combine a split
  // first piece left to the end of the range (-1: none), [15] step decisions ready, [16] the
  // status word the plan read, [17] STEP: the consumers have started the range's last piece,
  // [18] and [19] the first and last CTA holding a piece of stream [14]
  int* misc = reinterpret_cast<int*>(smem + lay.misc);
  uint32_t* bits = reinterpret_cast<uint32_t*>(smem + lay.bits);
  Partial<D>* slots = reinterpret_cast<Partial<D>*>(smem + lay.merge);
  int* prefix = reinterpret_cast<int*>(smem + lay.prefix);
  int* sid = reinterpret_cast<int*>(smem + lay.sid);
  // STEP, per call stream: retained count and tokens seen before the step, the logical
  // slot of the token leaving now (-1: none), the slot the new token takes (-1: not
  // appended), flags (1 pops a page, 2 alpha, 4 bad seq id, 8 stream full, 16 pool
  // exhausted) and the pop rank.
  int* s_nold = reinterpret_cast<int*>(smem + lay.step);
  int* s_pos = s_nold + a.S;
  int* s_rslot = s_pos + a.S;
  int* s_tslot = s_rslot + a.S;
  int* s_flag = s_tslot + a.S;
  int* s_rank = s_flag + a.S;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nst = a.n_seqs * a.hkv;
  volatile int* abort_flag = misc;
  // The status this launch acts on. A fused step of parity p reads the common
  // word and the step-error word of parity p (errors it finds itself go to the
  // other one); every other launch reads all of them.
  auto launch_status = [&]() -> int {
    if constexpr (STEP) {
      const int s0 = read_word(&a.ctrl[kCtrlStatus]);
      const int e = read_word(&a.ctrl[kCtrlStepErr + a.par]);
      return s0 != 0 ? s0 : e;
    } else {
      return read_status(a.ctrl);
    }
  };

  if (tid == 0) {
    if constexpr (MMA) prefetch_tensormap(&tmap);
    misc[0] = 0;
    misc[14] = -1;
    misc[15] = 0;
    misc[17] = 0;
    for (int s = 0; s < NCW * spw; ++s) mbar_init(smem_addr(&full[s]), 1);
    fence_mbar_init();
  }
  // The state parity the counts are read at: the host's, or (attention launched
  // into a stream under capture, a.par < 0) the cache's parity word, read with
  // the seq ids in the plan.
  int cpar = a.par;
  // Call streams [b0, e0) of this thread in the plan.
  const int per = (nst + kThreads - 1) / kThreads;
  const int b0 = min(tid * per, nst), e0 = min(b0 + per, nst);

  // STEP: the schedule the previous fused step left (counts, positions and
  // leaving slots after it, this CTA's page ids), trusted when the host says
  // no other call has changed the cache since.
  const unsigned long long trust = STEP ? a.step.trust : 0ull;
  const int tbuf = (int)(trust & 1ull);
  int4 thdr = make_int4(0, 0, 0, 0);   // header of this CTA's page list in it
  int spec_pg = 0;                     // consumer lanes: page id of the warp's job `lane` in it
  auto load_schedule_head = [&]() {
    const size_t cell = (size_t)tbuf * gridDim.x + blockIdx.x;
    thdr = ld_early4(a.step.next.hdr + 2 * cell);
    if (warp < NCW && warp + NCW * lane < a.step.next.cap)
      spec_pg = ld_early(a.step.next.list + cell * a.step.next.cap + warp + NCW * lane);
  };
  // This CTA's page ids come from the schedule when every stream of the call
  // matched it (same streams in the same order, hence the same counts and the
  // same partition) and its page list was written for exactly this call.
  auto list_matches = [&](long long P_, int ncta_, bool any_miss_) -> bool {
    const bool head = (unsigned long long)(uint32_t)thdr.x + ((unsigned long long)(uint32_t)thdr.y << 32) == trust &&
                      thdr.z == nst;
    thdr = make_int4(0, 0, 0, head ? thdr.w : -1);   // only the page count is needed from here on
    return STEP && trust != 0 && !any_miss_ && head && thdr.w == (int)P_ && ncta_ <= a.step.next.cap;
  };

  // STEP, early start. When the host knows that the kernel just before this
  // one in the stream does not write this cache, everything the schedule
  // describes (and the cache pages themselves) is final before the dependency
  // wait; only the call's own inputs (seq ids, alpha, queries, new rows) may
  // still be in the making. The plan and the first page copies then go ahead
  // of the wait on the guess that the call has the streams of the step that
  // wrote the schedule, which the seq ids confirm after it. This overlaps the
  // start of this launch with the end of the previous one.
  bool pre_ok = false;     // CTA-uniform: planned and copies issued before the wait
  bool any_miss = true;    // some stream of the call did not match the schedule
  int pre_k0 = 0, pre_k1 = 0;   // this CTA's range (in the guessed plan, then in the plan)
  using Query = typename std::conditional<MMA, MmaQuery<D>, SimtQuery<D>>::type;
  Query qcur;              // consumer lanes: the query of the piece about to start
  auto fetch_query = [&](int stream) {
    if constexpr (MMA) mma_fetch_q<D>(qcur, a, stream / a.hkv, stream % a.hkv, lane);
    else simt_fetch_q<D, E>(qcur, a, stream / a.hkv, stream % a.hkv, lane);
  };
  const PlanEntry* tentries = STEP ? a.step.next.entry + (size_t)tbuf * a.step.next.S : nullptr;
  if (STEP && trust != 0 && a.step.pre != 0) {
    load_schedule_head();
    const int4 trange = ld_early4(a.step.next.hdr + 2 * ((size_t)tbuf * gridDim.x + blockIdx.x) + 1);
    const int status = tid == 0 ? launch_status() : 0;
    const int free_depth = tid == 0 ? read_word(&a.ctrl[kCtrlFree + a.par]) : 0;
    bool miss = false;
    for (int i = b0; i < e0; ++i) {
      const int4 en = ld_early4(reinterpret_cast<const int4*>(tentries + i));
      const int4 e2 = ld_early4(reinterpret_cast<const int4*>(tentries + i) + 1);   // tag, first
      const unsigned long long etag = (unsigned long long)(uint32_t)e2.x | ((unsigned long long)(uint32_t)e2.y << 32);
      const bool ok = etag == trust && en.w >= 0 && en.w < a.max_seqs;
      const int nn = ok ? clamp_count(en.x, a.mps, a.ctrl) : 0;
      s_nold[i] = nn;
      s_pos[i] = en.y;
      s_flag[i] = 0;
      s_rslot[i] = ok && en.y >= a.step.dv.w && (en.z & 1) ? (en.z >> 1) : -1;
      sid[i] = ok ? en.w * a.hkv + i % a.hkv : 0;
      // The entries of one step hold the page offsets of its streams, so the
      // prefix needs no scan (any entry of another step drops the guess).
      prefix[i + 1] = ok ? e2.z + (nn + kPage - 1) / kPage : 0;
      miss |= !ok;
    }
    if (tid == 0) {
      prefix[0] = 0;
      misc[1] = (status == 0);
      misc[12] = free_depth;
      misc[16] = status;
    }
    any_miss = __syncthreads_or(miss) != 0;
    const long long P0 = prefix[nst];
    const int k0 = trange.x, k1 = trange.y;   // the range the step that wrote the list cut for this CTA
    pre_ok = misc[1] != 0 && list_matches(P0, k1 - k0, any_miss) && 0 <= k0 && k0 <= k1 && k1 <= P0;
    pre_k0 = k0;
    pre_k1 = k1;
    if (pre_ok && warp < NCW) {
      const int nj = k1 - k0 > warp ? (k1 - k0 - warp + NCW - 1) / NCW : 0;
      for (int j = 0; j < spw && j < nj; ++j) {
        int pg = __shfl_sync(0xffffffffu, spec_pg, j);
        if (lane == 0) {
          if (pg < 0 || pg >= a.max_pages) {
            latch(a.ctrl, DMS_ERR_INVALID);
            pg = 0;
          }
          issue_page<D, MMA, E>(full + warp * spw, smem + lay.stages + (size_t)warp * spw * kStage, spw, j, pg,
                                &tmap, a.kv);
        }
      }
    }
  }

  // Attention alone, early start: the same idea without a schedule. The
  // call's streams are guessed to be those of the previous attention call on
  // this cache (its list is left on the device); their counts, the page table
  // and the pages are cache state, final before the wait when the kernel before
  // this one does not write this cache. The guess is checked after the wait.
  int pid_pre = 0;   // consumer lanes: page id of the warp's job `lane` in the guessed plan
  if (!STEP && a.pre_attn) {   // (taken only when the host knows the parity: a.par >= 0)
    const int32_t* ncur = a.n + (size_t)cpar * a.n_stride;
    const int status = tid == 0 ? read_status(a.ctrl) : 0;
    const int gcount = ld_early(a.guess_rd);
    bool bad = false;
    int local = 0;
    for (int i = b0; i < e0; ++i) {
      const int seq = ld_early(a.guess_rd + 1 + i / a.hkv);   // within the buffer: n_seqs <= max_seqs
      int pages = 0, st = 0;
      if (seq < 0 || seq >= a.max_seqs) {
        bad = true;
      } else {
        st = seq * a.hkv + i % a.hkv;
        pages = (clamp_count(ld_early(ncur + st), a.mps, a.ctrl) + kPage - 1) / kPage;   // through L2
      }
      sid[i] = st;
      prefix[i + 1] = pages;
      local += pages;
    }
    int total;
    int run = block_exclusive_scan(local, misc + 3, &total);
    for (int i = b0; i < e0; ++i) {
      run += prefix[i + 1];
      prefix[i + 1] = run;
    }
    if (tid == 0) {
      prefix[0] = 0;
      misc[1] = (status == 0);
    }
    bad |= gcount != a.n_seqs;
    pre_ok = !__syncthreads_or(bad) && misc[1] != 0;
    if (pre_ok) {
      const Cut cut0(prefix[nst], nst, kX, gridDim.x);
      auto pf = [&](int i) -> long long { return prefix[i]; };
      pre_k0 = (int)cut0.begin(blockIdx.x, nst, pf);
      pre_k1 = (int)cut0.begin(blockIdx.x + 1, nst, pf);
      if (warp < NCW) {
        const int nj = pre_k1 - pre_k0 > warp ? (pre_k1 - pre_k0 - warp + NCW - 1) / NCW : 0;
        if (lane < nj) {
          const int kk = pre_k0 + warp + NCW * lane;
          const int i = stream_of(prefix, nst, kk);
          if (in_bounds(sid[i], (long long)a.max_seqs * a.hkv, a.ctrl) && in_bounds(kk - prefix[i], a.mps, a.ctrl))
            pid_pre = ld_early(a.page_table + (size_t)sid[i] * a.mps + (kk - prefix[i]));
          if (pid_pre < 0 || pid_pre >= a.max_pages) {
            latch(a.ctrl, DMS_ERR_INVALID);
            pid_pre = 0;
          }
        }
        for (int j = 0; j < spw && j < nj; ++j) {
          const int pg = __shfl_sync(0xffffffffu, pid_pre, j);
          if (lane == 0)
            issue_page<D, MMA, E>(full + warp * spw, smem + lay.stages + (size_t)warp * spw * kStage, spw, j, pg,
                                  &tmap, a.kv);
        }
      }
    }
  }

  // Launched early behind the previous kernel of the stream (programmatic
  // dependent launch): everything above overlaps it; nothing it writes is
  // read before this point.
  grid_dependency_wait();

  if (pre_ok) {
    // The call's seq ids against the guess, and (STEP) the alpha of its new
    // tokens, in the same round trip as the query of the CTA's first piece.
    if (warp < NCW && pre_k1 > pre_k0) fetch_query(stream_of(prefix, nst, pre_k0));
    bool bad = false;
    for (int i = b0; i < e0; ++i) {
      const int seq = a.seq_ids[i / a.hkv];
      if constexpr (STEP) {
        const int al = alpha_at(a.step.asrc, (size_t)(i / a.hkv), i % a.hkv);
        s_flag[i] = al != 0 ? 2 : 0;
      }
      bad |= seq != sid[i] / a.hkv;
    }
    if (__syncthreads_or(bad)) {
      // Another call: let the guessed copies land, then take every stage
      // barrier of the warp exactly two phases on with plain arrivals (one
      // after a landed copy, two on an unused stage), so that each is back at
      // a phase of parity 0 as the pipeline expects; then plan from the seq ids.
      if (warp < NCW && lane == 0) {
        const int nj = min(spw, pre_k1 - pre_k0 > warp ? (pre_k1 - pre_k0 - warp + NCW - 1) / NCW : 0);
        for (int j = 0; j < spw; ++j) {
          const uint32_t bar = smem_addr(&full[warp * spw + j]);
          if (j < nj) {
            mbar_wait_timed(bar, 0, a.ctrl);
          } else {
            mbar_arrive(bar);
          }
          mbar_arrive(bar);
        }
      }
      __syncthreads();   // every drain is done before the plan below
      pre_ok = false;
    }
  }

  // ---- plan: retained pages per stream of the call (prefix) and stream ids,
  // in smem. The status word is read in the same round trip as the seq ids.
  // STEP: so are the schedule entries (a stream whose entry does not match
  // falls back to the cache state) and this CTA's page ids from it.
  if (!pre_ok) {
    if (STEP && trust != 0) load_schedule_head();
    // Both control words are kept in registers until the loop's loads are out:
    // a shared-memory store of a loaded value here would hold them back one
    // round trip.
    const int status = tid == 0 ? launch_status() : 0;
    const int free_depth = (STEP && tid == 0) ? read_word(&a.ctrl[kCtrlFree + a.par]) : 0;
    // The current counts: the parity the host passed, else (a launch captured
    // into a graph) the cache's parity word, read in this round trip.
    if (cpar < 0) cpar = read_par(a.ctrl);
    const int32_t* ncur = a.n + (size_t)cpar * a.n_stride;
    bool miss = !STEP || trust == 0;
    int local = 0;
    for (int i = b0; i < e0; ++i) {
      const int seq = a.seq_ids[i / a.hkv];
      const int al = STEP ? alpha_at(a.step.asrc, (size_t)(i / a.hkv), i % a.hkv) : 0;   // same round trip as the seq id
      int4 en = make_int4(0, 0, 0, -1);
      unsigned long long etag = 0;
      if (STEP && trust != 0) {
        en = ld_early4(reinterpret_cast<const int4*>(tentries + i));
        etag = ld_early_u64(&tentries[i].tag);
      }
      int pages = 0, st = 0;
      if (seq < 0 || seq >= a.max_seqs) {
        if constexpr (STEP) {
          s_flag[i] = 4;   // latched once every CTA has read the status
          s_rslot[i] = -1;
        } else {
          latch(a.ctrl, DMS_ERR_BAD_SEQ);
        }
        miss = true;
      } else {
        st = seq * a.hkv + i % a.hkv;
        const bool hit = STEP && trust != 0 && etag == trust && en.w == seq;
        const int nn = clamp_count(hit ? en.x : ncur[st], a.mps, a.ctrl);
        pages = (nn + kPage - 1) / kPage;
        if constexpr (STEP) {
          const int ps = hit ? en.y : a.step.dv.pos[(size_t)cpar * a.step.dv.S + st];
          s_nold[i] = nn;
          s_pos[i] = ps;
          s_flag[i] = al != 0 ? 2 : 0;
          // The token at ps - w leaves now if it was marked; unknown until the
          // window ring is read when the schedule had no entry.
          s_rslot[i] = hit ? ((ps >= a.step.dv.w && (en.z & 1)) ? (en.z >> 1) : -1) : kRslotUnknown;
        }
        miss |= !hit;
      }
      sid[i] = st;
      prefix[i + 1] = pages;
      local += pages;
    }
    int total;
    int run = block_exclusive_scan(local, misc + 3, &total);
    for (int i = b0; i < e0; ++i) {
      run += prefix[i + 1];
      prefix[i + 1] = run;
    }
    if (tid == 0) {
      prefix[0] = 0;
      misc[1] = (status == 0);
      misc[16] = status;
      if (STEP) misc[12] = free_depth;
    }
    any_miss = __syncthreads_or(miss) != 0;
    // This CTA's range (before any query fragment is held: the search needs registers).
    const Cut cut(prefix[nst], nst, kX, gridDim.x);
    auto pf = [&](int i) -> long long { return prefix[i]; };
    pre_k0 = (int)cut.begin(blockIdx.x, nst, pf);
    pre_k1 = (int)cut.begin(blockIdx.x + 1, nst, pf);
  }
  grid_dependents_launch();   // the next kernel may queue up behind this one
  if (STEP && tid == 0) misc[3] = 0;   // written by the step warp late in the launch
  if (!STEP && a.guess_wr && blockIdx.x == 0) {   // this call's stream list, the next call's guess
    for (int b = tid; b < a.n_seqs; b += kThreads) a.guess_wr[1 + b] = a.seq_ids[b];
    if (tid == 0) a.guess_wr[0] = a.n_seqs;
  }
  const bool healthy = misc[1] != 0;
  if constexpr (!STEP) {
    if (!healthy) return;   // poisoned cache: do nothing (uniform over the CTA)
  }
  const int G = gridDim.x;
  if constexpr (!STEP) {
    // Streams with nothing retained produce zeros.
    for (int i = blockIdx.x; i < nst; i += G) {
      if (prefix[i + 1] != prefix[i]) continue;
      const int b = i / a.hkv, kvh = i % a.hkv;
      for (int e = tid; e < a.g * D; e += kThreads) store_out(a, b, kvh * a.g + e / D, e % D, D, 0.f);
    }
  }
  const int K0 = healthy ? pre_k0 : 0, K1 = healthy ? pre_k1 : 0;
  const bool has_range = K1 > K0;
  if constexpr (!STEP) {
    if (!has_range) return;   // uniform over the CTA
  }
  const int ncta = K1 - K0;
  const bool list_ok = pre_ok || list_matches(prefix[nst], ncta, any_miss);   // called once: it narrows thdr
  int consumed = 0, issued = 0;
  uint64_t* myfull = full + (warp < NCW ? warp : 0) * spw;

  if (STEP && warp == NCW) {
    step_warp<D, E, kX>(a, nst, prefix, sid, s_nold, s_pos, s_rslot, s_tslot, s_flag, s_rank, misc, bits, healthy,
                    abort_flag, K0, K1);
  } else if (STEP || has_range) {
    // ---- this warp's page pipeline: CTA pages c = warp + NCW * j, j = 0 .. njobs-1
    const int njobs = has_range && ncta > warp ? (ncta - warp + NCW - 1) / NCW : 0;
    uint8_t* mystage = smem + lay.stages + (size_t)warp * spw * kStage;
    const int32_t* tlist = STEP ? a.step.next.list + ((size_t)tbuf * gridDim.x + blockIdx.x) * a.step.next.cap
                                : nullptr;
    auto checked = [&](int pg) -> int {
      if (pg < 0 || pg >= a.max_pages) {
        latch(a.ctrl, DMS_ERR_INVALID);
        pg = 0;
      }
      return pg;
    };
    auto lookup = [&](int j) -> int {   // physical page of the warp's j-th page
      if (j >= njobs) return 0;
      if (STEP && list_ok) return checked(__ldg(tlist + warp + NCW * j));
      const int kk = K0 + warp + NCW * j;
      const int i = stream_of(prefix, nst, kk);
      if (!in_bounds(sid[i], (long long)a.max_seqs * a.hkv, a.ctrl) || !in_bounds(kk - prefix[i], a.mps, a.ctrl))
        return 0;
      return checked(__ldg(a.page_table + (size_t)sid[i] * a.mps + (kk - prefix[i])));
    };
    using State = typename std::conditional<MMA, MmaState<D>, SimtState<D>>::type;
    State S;
    auto start_piece = [&]() {   // take the fetched query, clear the softmax state
      if constexpr (MMA) mma_start<D>(S, qcur);
      else simt_start<D>(S, qcur);
    };
    auto load_query = [&](int stream) {
      fetch_query(stream);
      start_piece();
    };
    // The first piece's query is requested in the same round trip as the page
    // ids, before the copies fill the memory queues.
    int i = has_range ? stream_of(prefix, nst, K0) : 0;
    if (has_range && !pre_ok) fetch_query(i);   // else fetched with the seq ids
    // STEP: the window-ring entry of every call stream (the token at s - w),
    // requested before the page ids so that both land before the first copies
    // are issued: a load queued behind the grid's first burst of page copies
    // waits microseconds.
    constexpr int kRingPer = (kStepMaxStreams + kMergeThreads - 1) / kMergeThreads;
    int ring_v[STEP ? kRingPer : 1];
    if (STEP && !pre_ok) {   // (the guessed plan knows every leaving slot)
#pragma unroll
      for (int q = 0; q < kRingPer; ++q) {
        const int il = tid + q * kMergeThreads;
        ring_v[q] = (il < nst && s_rslot[il] == kRslotUnknown)
                        ? ld_early(a.step.dv.ring + ring_leaving(a.step.dv, sid[il], s_pos[il]))
                        : 0;
      }
    }
    int jb = 0;   // page ids of jobs [jb, jb+32) in pid_cur, [jb+32, jb+64) in pid_nxt
    int pid_cur = (STEP && list_ok) ? (lane < njobs ? checked(spec_pg) : 0)
                  : (!STEP && pre_ok) ? pid_pre   // looked up before the wait
                                      : lookup(lane);
    int pid_nxt = lookup(32 + lane);
    auto issue = [&](int j) {   // warp-uniform; j = issued
      if (j - jb >= 32) {
        pid_cur = pid_nxt;
        jb += 32;
        pid_nxt = lookup(jb + 32 + lane);
      }
      const int r = j - jb;
      const int pg = __shfl_sync(0xffffffffu, r < 32 ? pid_cur : pid_nxt, r & 31);
      if (lane == 0) issue_page<D, MMA, E>(myfull, mystage, spw, j, pg, &tmap, a.kv);
      issued = j + 1;
    };
    if (pre_ok) {
      issued = min(spw, njobs);   // the first copies went out before the dependency wait
    } else {
      for (int j = 0; j < spw && j < njobs; ++j) issue(j);
    }
    if constexpr (STEP) {
      // The logical slot of the token leaving at this step (-1: none), for the
      // consumers' masks and the step warp's decisions.
      if (!pre_ok) {
#pragma unroll
        for (int q = 0; q < kRingPer; ++q) {
          const int il = tid + q * kMergeThreads;
          if (il < nst && s_rslot[il] == kRslotUnknown)
            s_rslot[il] = (s_pos[il] >= a.step.dv.w && (ring_v[q] & 1)) ? (ring_v[q] >> 1) : -1;
        }
      }
      // Hand them to the step warp (which syncs on barrier 2). A consumer masks
      // with the slots other consumer threads resolved, so when any was read from
      // the ring here the consumers wait for all of them too (CTA-uniform).
      if (!pre_ok && any_miss) named_barrier(2, kThreads);
      else named_barrier_arrive(2, kThreads);
    }
    if (has_range) {


      const int32_t* ncur = a.n + (size_t)cpar * a.n_stride;
      auto retained_of = [&](int stream) -> int {   // retained count the attention runs over
        if constexpr (STEP) return s_nold[stream];
        else return clamp_count(__ldg(ncur + sid[stream]), a.mps, a.ctrl);
      };
      const MmaOffsets<D> off(lane);
      int k = K0;
      start_piece();
      int nn = retained_of(i);
      bool decisions = false;   // STEP: the step warp's decisions have been seen
      auto await_decisions = [&]() {
        if (STEP && !decisions) {
          if (lane == 0) wait_flag_ge(misc + 15, 1, abort_flag, a.ctrl);
          __syncwarp();
          __threadfence_block();
          decisions = true;
        }
      };
      while (k < K1) {
        const int pstart = prefix[i], pend = prefix[i + 1];
        const int pe = min(pend, K1);
        const int b = i / a.hkv, kvh = i % a.hkv;
        const bool whole = (k == pstart) && (pe == pend);
        // STEP: tell the step warp the range's last piece has begun (it then reads
        // whether the stream's other pieces are all published).
        if (STEP && pe == K1 && tid == 0) *reinterpret_cast<volatile int*>(&misc[17]) = 1;
        const int rslot = STEP ? s_rslot[i] : -1;   // row of the token leaving at this step
        auto rows_of = [&](int p) -> uint32_t {      // rows to attend in page p of the stream
          const int valid = (pstart + p == pend - 1) ? nn - kPage * p : kPage;
          uint32_t r = valid >= kPage ? 0xffffu : ((1u << valid) - 1u);
          if (rslot >= 0 && (rslot >> 4) == p) r &= ~(1u << (rslot & 15));
          return r;
        };

        const int rel = k - K0;
        for (int c = rel + ((warp - rel) % NCW + NCW) % NCW; c < pe - K0;) {
          const int j = (c - warp) / NCW;
          const int nb = (NB == 2 && c + NCW < pe - K0) ? 2 : 1;   // pages in this batch (same stream)
          bool ok = mbar_wait_bounded(smem_addr(&myfull[j % spw]), (j / spw) & 1, abort_flag, a.ctrl);
          if (nb == 2) ok &= mbar_wait_bounded(smem_addr(&myfull[(j + 1) % spw]), ((j + 1) / spw) & 1, abort_flag, a.ctrl);
          if (ok) {
            const int p = K0 + c - pstart;   // page index within the stream
            const uint8_t* st0 = mystage + (size_t)(j % spw) * kStage;
            if constexpr (MMA) {
              if (nb == 2) {
                const uint32_t stg[2] = {smem_addr(st0), smem_addr(mystage + (size_t)((j + 1) % spw) * kStage)};
                const uint32_t rw[2] = {rows_of(p), rows_of(p + NCW)};
                mma_pages<D, 2>(S, stg, rw, a.sl2e, lane, off);
              } else {
                const uint32_t stg[1] = {smem_addr(st0)};
                const uint32_t rw[1] = {rows_of(p)};
                mma_pages<D, 1>(S, stg, rw, a.sl2e, lane, off);
              }
            } else {
              simt_page<D, E>(S, reinterpret_cast<const E*>(st0), rows_of(p), a.g, lane);
            }
          }
          consumed = j + nb;
          __syncwarp();
          const bool stop = __any_sync(0xffffffffu, *abort_flag != 0);
          for (int q = 0; q < nb; ++q)
            if (j + q + spw < njobs && !stop) issue(j + q + spw);
          c += nb * NCW;
        }

        // ---- end of the piece: merge the warps' states in shared memory
        if constexpr (MMA) mma_to_slot<D>(S, &slots[warp], lane);
        else simt_to_slot<D>(S, &slots[warp], lane);
        // start loading the next piece's query while the CTA merges
        const int inext = pe < K1 ? stream_of(prefix, nst, pe) : i;
        if (pe < K1) load_query(inext);
        const int nn_next = pe < K1 ? retained_of(inext) : 0;
        // STEP, the range's last piece of a split stream: whether the step warp
        // has seen every other piece of it published (one snapshot for all).
        if (STEP && tid == 0 && !whole && pe == K1) misc[4] = *reinterpret_cast<volatile int*>(&misc[3]) == 1;
        // Merge: thread t owns query head h = t / (D/4) and dims [4 d4, 4 d4 + 4);
        // the CTA's result for its items stays in registers for the combine.
        constexpr int kItems = kMaxGroup * D / 4;
        constexpr int kIters = (kItems + kMergeThreads - 1) / kMergeThreads;
        const int items = a.g * (D / 4);
        named_barrier(1, kMergeThreads);
        // (read from shared memory where it is used: a register held across the merge spills)
        auto known_last = [&]() -> bool {
          return STEP && !whole && pe == K1 && *reinterpret_cast<volatile int*>(&misc[4]) != 0;
        };

        // The step warp's decisions are needed only by a merge that may finish
        // its stream (a whole piece, or the range's last piece, which may
        // combine); a split first piece only publishes its partial.
        const bool may_finish = whole || pe == K1;
        if (STEP && may_finish) await_decisions();
        const bool add_new = STEP && may_finish && s_tslot[i] >= 0;   // the stream's new token (appended by this step)
        float4 myO[kIters];
        float myM[kIters], myL[kIters];
        Partial<D>* part = reinterpret_cast<Partial<D>*>(a.part) +
                           (in_bounds(blockIdx.x + i, a.part_slots, a.ctrl) ? blockIdx.x + i : 0);
#pragma unroll
        for (int it = 0; it < kIters; ++it) {
          const int t = tid + it * kMergeThreads;
          const bool live = t < items;
          if (!__any_sync(0xffffffffu, live)) break;   // warp-uniform
          const int h = (live ? t : 0) / (D / 4), d4 = (live ? t : 0) % (D / 4);
          float M = -INFINITY;
#pragma unroll
          for (int w = 0; w < NCW; ++w) M = fmaxf(M, slots[w].m[h]);
          float L = 0.f;
          float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int w = 0; w < NCW; ++w) {
            // 0 for a warp that saw nothing (m = -inf); all 0 if no warp saw a token
            const float sc = M == -INFINITY ? 0.f : ex2(slots[w].m[h] - M);
            const float4 o = *reinterpret_cast<const float4*>(&slots[w].O[h][4 * d4]);
            L = fmaf(slots[w].l[h], sc, L);
            O.x = fmaf(o.x, sc, O.x);
            O.y = fmaf(o.y, sc, O.y);
            O.z = fmaf(o.z, sc, O.z);
            O.w = fmaf(o.w, sc, O.w);
          }
          if (whole) {
            if constexpr (STEP) add_new_token<D, E>(a, i, h, d4, add_new, M, L, O);   // warp-collective
            if (live) store_out4(a, b, kvh * a.g + h, 4 * d4, D, O, L > 0.f ? 1.f / L : 0.f);
          } else if (live) {
            if (!known_last()) {   // else nobody reads it: this CTA combines the stream
              __stcg(reinterpret_cast<float4*>(&part->O[h][4 * d4]), O);
              if (d4 == 0) {
                __stcg(&part->m[h], M);
                __stcg(&part->l[h], L);
              }
            }
            myO[it] = O;
            myM[it] = M;
            myL[it] = L;
          }
        }
        named_barrier(1, kMergeThreads);   // the slots are read and the partial (if any) is complete
        if (!whole) {
          // Publish the partial: the CTA's stores, ordered by the barrier, are
          // released by thread 0's device-scope add; the adder that completes the
          // count acquires every other piece and combines.
          const Cut cut(prefix[nst], nst, kX, G);   // (from shared memory: nothing held across the pieces)
          const int first = cut.owner(pstart, i), last = cut.owner(pend - 1, i);
          if (pe < K1) {
            // A split piece inside the range is its first piece. Thread 0
            // publishes it while the CTA goes on; a combine it finds due is done
            // by the whole CTA at the end of the range.
            if (tid == 0 && atomic_add_acq_rel_gpu(&a.cnt[i], 1) == last - first) {
              misc[14] = i;
              misc[18] = first;
              misc[19] = last;
            }
          } else {
            const bool shortcut = known_last();
            if (shortcut) {
              __threadfence_block();   // the step warp's acquire of the other pieces, passed on
            } else {
              if (tid == 0) misc[2] = (atomic_add_acq_rel_gpu(&a.cnt[i], 1) == last - first);
              named_barrier(1, kMergeThreads);
            }
            if (shortcut || misc[2]) {
              const Partial<D>* base = reinterpret_cast<const Partial<D>*>(a.part) + i;
              const int me = blockIdx.x;
              const int last_ok = in_bounds((long long)last + i, a.part_slots, a.ctrl) ? last : first - 1;
#pragma unroll
              for (int it = 0; it < kIters; ++it) {
                const int t = tid + it * kMergeThreads;
                const bool live = t < items;
                if (!__any_sync(0xffffffffu, live)) break;   // warp-uniform
                const int h = (live ? t : 0) / (D / 4), d4 = (live ? t : 0) % (D / 4);
                NewTok nt;   // tensor-core kernel: in flight with the partials (the CUDA-core one has no registers to spare)
                if constexpr (STEP && MMA) fetch_new_token<D, E>(a, i, h, d4, nt);
                float M = live ? myM[it] : 0.f, L = live ? myL[it] : 1.f;
                float4 O = live ? myO[it] : make_float4(0.f, 0.f, 0.f, 0.f);
                for (int c0 = first; c0 <= last_ok; c0 += 4) {   // loads of 4 pieces in flight at once
                  float mc[4], lc[4];
                  float4 oc[4];
#pragma unroll
                  for (int u = 0; u < 4; ++u) {
                    const int c = c0 + u;
                    const bool use = c <= last_ok && c != me;
                    mc[u] = use ? __ldcg(&base[c].m[h]) : -INFINITY;
                    lc[u] = use ? __ldcg(&base[c].l[h]) : 0.f;
                    oc[u] = use ? __ldcg(reinterpret_cast<const float4*>(&base[c].O[h][4 * d4]))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
                  }
#pragma unroll
                  for (int u = 0; u < 4; ++u) merge_into(M, L, O, mc[u], lc[u], oc[u]);
                }
                if constexpr (STEP && MMA) apply_new_token<D>(nt, a.sl2e, add_new, M, L, O);   // warp-collective
                else if constexpr (STEP) add_new_token<D, E>(a, i, h, d4, add_new, M, L, O);
                if (live) store_out4(a, b, kvh * a.g + h, 4 * d4, D, O, L > 0.f ? 1.f / L : 0.f);
              }
              if (tid == 0) a.cnt[i] = 0;   // ready for the next launch (stream order)
            }
          }
        }
        k = pe;
        i = inext;
        nn = nn_next;
      }
    }
  }

  // ---- a split first piece that completed its stream: combine all its pieces
  __syncthreads();
  if (tid < kMergeThreads && misc[14] >= 0) {
    const int i = misc[14], first = misc[18], last = misc[19];
    combine_stream<D, E, STEP>(a, i, first, last, tid, kMergeThreads, STEP && s_tslot[i] >= 0);
    if (tid == 0) a.cnt[i] = 0;   // ready for the next launch (stream order)
  }

  // Drain: copies issued but not consumed (only after an abort) must land before exit.
  if (warp < NCW && lane == 0)
    for (int j = consumed; j < issued; ++j) mbar_wait_timed(smem_addr(&myfull[j % spw]), (j / spw) & 1, a.ctrl);
}

// ---------------------------------------------------------------------------
// Kernel table.

using KernelFn = void (*)(const AttnArgs, const __grid_constant__ CUtensorMap);

template <int D, int NCW, int NB, bool MMA, typename E, bool STEP>
KernelFn kernel_ptr() { return attn_kernel<D, NCW, NB, MMA, E, STEP>; }

template <int NB, bool MMA, typename E, bool STEP>
KernelFn pick_ncw(int d, int ncw) {
  if (d == 64) return ncw == 4 ? kernel_ptr<64, 4, NB, MMA, E, STEP>() : kernel_ptr<64, 8, NB, MMA, E, STEP>();
  return ncw == 4 ? kernel_ptr<128, 4, NB, MMA, E, STEP>() : kernel_ptr<128, 8, NB, MMA, E, STEP>();
}

template <bool STEP>
KernelFn pick_kernel(int d, int dtype, int kernel, int ncw, int nb) {
  if (kernel == DMS_ATTN_MMA)
    return nb == 2 ? pick_ncw<2, true, uint16_t, STEP>(d, ncw) : pick_ncw<1, true, uint16_t, STEP>(d, ncw);
  if (dtype == DMS_BF16) return pick_ncw<1, false, uint16_t, STEP>(d, ncw);
  return pick_ncw<1, false, float, STEP>(d, ncw);
}

// Launch-shape overrides for tuning sweeps. Only a build with DMS_TUNING defined
// reads them; the library as shipped always takes the defaults, which are the
// shapes its tests cover.
int env_int(const char* name, int dflt) {
#ifdef DMS_TUNING
  const char* v = getenv(name);
  return (v && *v) ? atoi(v) : dflt;
#else
  (void)name;
  return dflt;
#endif
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);


cudaError_t prepare(const Dev& dv, int dtype, int kernel_choice, int num_sms, bool step, AttnPlan* plan) {
  int kernel = kernel_choice;
  if (kernel == DMS_ATTN_AUTO) kernel = (dtype == DMS_BF16) ? DMS_ATTN_MMA : DMS_ATTN_SIMT;
  if (kernel == DMS_ATTN_MMA && dtype != DMS_BF16) return cudaErrorInvalidValue;
  // Tuning overrides: warps per CTA (4, 8), CTAs per SM (1, 2), stages per warp,
  // pages per warp iteration (1, 2; tensor-core kernel only).
  int ncw = env_int("DMS_ATTN_WARPS", 8);
  if (ncw != 4) ncw = 8;
  const int nb = (kernel == DMS_ATTN_MMA && env_int("DMS_ATTN_BATCH", 2) != 1) ? 2 : 1;
  const int ctas = env_int("DMS_ATTN_CTAS", 1) == 2 ? 2 : 1;
  const int stage_bytes = 2 * kPage * dv.d * dv.elem_bytes;
  int dev = 0, per_sm_smem = 0, per_block_smem = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&per_sm_smem, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&per_block_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  const int budget = std::min(per_block_smem, per_sm_smem / ctas - 1024);   // 1 KB per CTA stays reserved
  const int fixed = smem_layout(ncw, 0, stage_bytes, dv.d, dv.S, step).total;
  int spw = std::min(8, (budget - fixed) / (ncw * stage_bytes));
  const int want = env_int("DMS_ATTN_STAGES", 0);
  if (want > 0) spw = std::min(spw, want);
  if (spw < nb) return cudaErrorInvalidConfiguration;

  KernelFn fn = step ? pick_kernel<true>(dv.d, dtype, kernel, ncw, nb) : pick_kernel<false>(dv.d, dtype, kernel, ncw, nb);
  plan->kernel = kernel;
  plan->ncw = ncw;
  plan->spw = spw;
  plan->fn = reinterpret_cast<void*>(fn);
  plan->threads = (ncw + (step ? 1 : 0)) * 32;
  plan->smem = (size_t)smem_layout(ncw, spw, stage_bytes, dv.d, dv.S, step).total;
  // The dynamic shared-memory limit is an attribute of the kernel function,
  // shared by every plan (every cache, every allocation-free call) that uses this
  // instantiation. It is set to the device's opt-in maximum, which every plan
  // fits under, so no plan's set-up can shrink the limit under another's launch.
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, fn);
  if (e != cudaSuccess) return e;
  const int limit = per_block_smem - (int)fa.sharedSizeBytes;
  if ((int)plan->smem > limit) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, limit);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, plan->threads, plan->smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  plan->grid = num_sms * std::min(per_sm, ctas);

  memset(&plan->tmap, 0, sizeof(plan->tmap));
  if (kernel == DMS_ATTN_MMA) {
    void* enc = nullptr;
    cudaDriverEntryPointQueryResult q;
    e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &enc, cudaEnableDefault, &q);
    if (e != cudaSuccess || enc == nullptr || q != cudaDriverEntryPointSuccess) return cudaErrorNotSupported;
    // Pool viewed as [max_pages][32 rows][d] bf16; box = 64 columns x 32 rows of one page.
    const cuuint64_t dims[3] = {(cuuint64_t)dv.d, 32, (cuuint64_t)dv.max_pages};
    const cuuint64_t strides[2] = {(cuuint64_t)dv.d * 2, (cuuint64_t)dv.d * 2 * 32};
    const cuuint32_t box[3] = {64, 32, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = reinterpret_cast<EncodeTiledFn>(enc)(
        &plan->tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, dv.kv, dims, strides, box, estr,
        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}


}  // namespace

cudaError_t attention_prepare(const Dev& dv, int dtype, int kernel_choice, int num_sms, AttnPlan* plan) {
  return prepare(dv, dtype, kernel_choice, num_sms, false, plan);
}

cudaError_t step_prepare(const Dev& dv, int dtype, int kernel_choice, int num_sms, AttnPlan* plan) {
  return prepare(dv, dtype, kernel_choice, num_sms, true, plan);
}

namespace {

AttnArgs attn_args(const Dev& dv, const AttnPlan& plan, int n_seqs, const int32_t* seq_ids, const void* Q,
                   int hq, float scale, void* out, int out_f32, const AttnCounts& counts) {
  AttnArgs a;
  memset(&a, 0, sizeof(a));
  a.seq_ids = seq_ids;
  a.Q = (const uint8_t*)Q;
  a.out = (uint8_t*)out;
  a.n = counts.n;
  a.n_stride = counts.stride;
  a.par = counts.par;
  a.page_table = dv.page_table;
  a.kv = dv.kv;
  a.ctrl = dv.ctrl;
  a.part = dv.part;
  a.cnt = dv.cnt;
  a.part_slots = dv.part_slots;
  a.n_seqs = n_seqs;
  a.hkv = dv.hkv;
  a.g = hq / dv.hkv;
  a.hq = hq;
  a.mps = dv.mps;
  a.max_seqs = dv.max_seqs;
  a.max_pages = dv.max_pages;
  a.out_f32 = out_f32;
  a.sl2e = scale * kLog2e;
  a.spw = plan.spw;
  a.S = dv.S;
  return a;
}

}  // namespace

cudaError_t launch_attention(const Dev& dv, const AttnPlan& plan, cudaStream_t st, int n_seqs,
                             const int32_t* seq_ids, const void* Q, int hq, float scale, void* out,
                             int out_f32, const AttnCounts& counts, const AttnGuess& guess) {
  if (n_seqs == 0) return cudaSuccess;
  AttnArgs a = attn_args(dv, plan, n_seqs, seq_ids, Q, hq, scale, out, out_f32, counts);
  a.guess_rd = guess.rd;
  a.guess_wr = guess.wr;
  // The early plan reads the counts before the dependency wait: only with the parity known.
  a.pre_attn = guess.early && guess.rd && guess.wr && counts.par >= 0 ? 1 : 0;
  return launch_dependent(reinterpret_cast<KernelFn>(plan.fn), dim3(plan.grid), dim3(plan.threads), plan.smem, st,
                          a, plan.tmap);
}

cudaError_t launch_step(const Dev& dv, const AttnPlan& plan, cudaStream_t st, int n_seqs, const int32_t* seq_ids,
                        const void* K, const void* V, const AlphaChoice& alpha, const void* Q, int hq,
                        float scale, void* out, int out_f32, int par, const NextPlan& next,
                        unsigned long long trust_tag, unsigned long long write_tag, bool early) {
  // Every launch flips the cache's state parity, so an empty call must not get here
  // (the host would count a flip that never happens).
  if (n_seqs <= 0) return cudaErrorInvalidValue;
  // A schedule is read from the buffer of its tag's parity and written to the
  // other one, so the two tags must be consecutive.
  if (write_tag == 0 || (trust_tag != 0 && trust_tag + 1 != write_tag)) return cudaErrorInvalidValue;
  if (par != 0 && par != 1) return cudaErrorInvalidValue;
  AttnArgs a = attn_args(dv, plan, n_seqs, seq_ids, Q, hq, scale, out, out_f32, AttnCounts{dv.n, dv.S, par});
  a.step.K = (const uint8_t*)K;
  a.step.V = (const uint8_t*)V;
  if (alpha.channel < 0) a.step.asrc = alpha_given(alpha.alpha, dv.hkv);
  else if (alpha.q_head < 0) a.step.asrc = alpha_from_keys(K, dv.hkv, dv.d, alpha.channel, dv.elem_bytes);
  else a.step.asrc = alpha_from_queries(Q, dv.hkv, hq / dv.hkv, dv.d, alpha.q_head, alpha.channel, dv.elem_bytes);
  a.step.dv = dv;
  a.step.next = next;
  a.step.trust = next.entry ? trust_tag : 0ull;
  a.step.wtag = write_tag;
  a.step.pre = early ? 1 : 0;
  return launch_dependent(reinterpret_cast<KernelFn>(plan.fn), dim3(plan.grid), dim3(plan.threads), plan.smem, st,
                          a, plan.tmap);
}

}  // namespace dms
