// dms_noalloc.cu - decode attention over caller-owned paged K/V with the
// split-K scratch in a static device array: the call allocates nothing.
//
// Who needs it: code that may not call cudaMalloc while it decodes, e.g.
// a host framework whose caching allocator already holds the device memory
// (a stray cudaMalloc may fail or synchronise the device), or a runtime that
// owns every buffer and lends the library only its K/V pages. Such a caller
// keeps the pool, the page table and the retained counts in its own memory
// and passes them in; the partial results and arrival counters that split-K
// needs live in g_scratch below, which the CUDA runtime places when it loads
// the library on a device and keeps until the process exits.
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "dms_internal.cuh"

namespace dms {
namespace {

// One piece's partial: [8 heads][d + 2] floats at d = 128.
constexpr size_t kPieceBytes = (size_t)kMaxGroup * (128 + 2) * sizeof(float);
constexpr size_t kCtrlBytes = 256;                                   // status word and spare control words
constexpr size_t kCountBytes = (size_t)DMS_NOALLOC_MAX_STREAMS * 4;  // per-stream arrival counters
constexpr size_t kPartOffset = kCtrlBytes + kCountBytes;             // 256-aligned
constexpr size_t kScratchBytes = kPartOffset + (size_t)DMS_NOALLOC_MAX_PIECES * kPieceBytes;
static_assert(kPartOffset % 256 == 0, "partials must start 256-aligned");

// Shared by every call on a device. Host code must not pass this name to a
// kernel: on the host it is a stand-in object, not a device address.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
constexpr int kPlans = 8;   // launch plans kept per device

// A launch plan and what it was made for (the tensor map holds the pool's
// address and size; the shared-memory plan arrays are sized by the streams).
struct CachedPlan {
  bool valid = false;
  unsigned long long used = 0;   // last use, for replacement
  AttnPlan plan;
  const void* pool = nullptr;
  int d = 0, dtype = 0, streams = 0, max_pages = 0;
};

// Per-device set-up, done by the first call on that device, and the plans of
// the last few distinct call shapes, so that a caller alternating between
// batch sizes or pools does not prepare a plan on every call.
struct DeviceState {
  bool ready = false;
  unsigned char* scratch = nullptr;   // device address of g_scratch
  int num_sms = 0;
  unsigned long long clock = 0;
  CachedPlan plans[kPlans];
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

int elem_bytes_of(int dtype) { return dtype == DMS_BF16 ? 2 : 4; }

}  // namespace
}  // namespace dms

static dms_status noalloc_impl(cudaStream_t stream, const dms_paged_kv* kv, int32_t n_seqs,
                                 const int32_t* seq_ids, const void* Q, int32_t num_q_heads,
                                 float scale, void* out, dms_dtype out_dtype) {
  using namespace dms;
  if (!kv || n_seqs < 0) return DMS_ERR_INVALID;
  const int hkv = kv->num_kv_heads, d = kv->head_dim;
  if (hkv < 1 || (d != 64 && d != 128)) return DMS_ERR_INVALID;
  if (kv->dtype != DMS_BF16 && kv->dtype != DMS_F32) return DMS_ERR_INVALID;
  if (out_dtype != DMS_BF16 && out_dtype != DMS_F32) return DMS_ERR_INVALID;
  if (kv->max_seqs < 1 || kv->max_pages < 1 || kv->max_pages_per_stream < 1) return DMS_ERR_INVALID;
  if (n_seqs > kv->max_seqs) return DMS_ERR_INVALID;
  if (num_q_heads < hkv || num_q_heads % hkv != 0 || num_q_heads / hkv > kMaxGroup) return DMS_ERR_INVALID;
  const long long nst = (long long)n_seqs * hkv;
  if (nst > DMS_NOALLOC_MAX_STREAMS) return DMS_ERR_INVALID;   // beyond the static scratch
  if (n_seqs == 0) return DMS_OK;
  auto aligned16 = [](const void* p) { return ((uintptr_t)p & 15u) == 0; };
  if (!kv->kv_pool || !kv->page_table || !kv->retained || !seq_ids || !Q || !out) return DMS_ERR_INVALID;
  if (!aligned16(kv->kv_pool) || !aligned16(Q) || !aligned16(out)) return DMS_ERR_INVALID;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DMS_ERR_CUDA;

  Dev dv;
  memset(&dv, 0, sizeof(dv));
  dv.n = const_cast<int32_t*>(kv->retained);
  dv.page_table = const_cast<int32_t*>(kv->page_table);
  dv.kv = reinterpret_cast<uint8_t*>(const_cast<void*>(kv->kv_pool));
  dv.S = (int)nst;   // sizes the kernel's per-call plan arrays in shared memory
  dv.hkv = hkv;
  dv.d = d;
  dv.mps = kv->max_pages_per_stream;
  dv.max_pages = kv->max_pages;
  dv.max_seqs = kv->max_seqs;
  dv.elem_bytes = elem_bytes_of(kv->dtype);

  AttnPlan plan;
  unsigned char* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState& ds = g_dev[dev];
    if (!ds.ready) {
      // The device address of the static array; valid for this device only.
      if (cudaGetSymbolAddress(reinterpret_cast<void**>(&ds.scratch), g_scratch) != cudaSuccess) return DMS_ERR_CUDA;
      if (cudaDeviceGetAttribute(&ds.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return DMS_ERR_CUDA;
      ds.ready = true;
    }
    CachedPlan* hit = nullptr;
    CachedPlan* victim = &ds.plans[0];
    for (CachedPlan& c : ds.plans) {
      if (c.valid && c.pool == kv->kv_pool && c.d == d && c.dtype == (int)kv->dtype && c.streams == (int)nst &&
          c.max_pages == kv->max_pages) {
        hit = &c;
        break;
      }
      if (!c.valid || (victim->valid && c.used < victim->used)) victim = &c;
    }
    if (hit == nullptr) {
      victim->valid = false;
      cudaError_t e = attention_prepare(dv, kv->dtype, DMS_ATTN_AUTO, ds.num_sms, &victim->plan);
      if (e != cudaSuccess) return e == cudaErrorInvalidValue ? DMS_ERR_INVALID : DMS_ERR_CUDA;
      victim->valid = true;
      victim->pool = kv->kv_pool;
      victim->d = d;
      victim->dtype = (int)kv->dtype;
      victim->streams = (int)nst;
      victim->max_pages = kv->max_pages;
      hit = victim;
    }
    hit->used = ++ds.clock;
    plan = hit->plan;
    scratch = ds.scratch;
  }
  // Every piece of a split stream needs a partial slot: (CTA, stream) pairs
  // map to CTA index + stream index, so the grid plus the streams must fit.
  if ((size_t)plan.grid + (size_t)nst > (size_t)DMS_NOALLOC_MAX_PIECES) return DMS_ERR_INVALID;

  dv.ctrl = reinterpret_cast<int32_t*>(scratch);
  dv.cnt = reinterpret_cast<int32_t*>(scratch + kCtrlBytes);
  dv.part = reinterpret_cast<float*>(scratch + kPartOffset);
  dv.part_slots = DMS_NOALLOC_MAX_PIECES;
  // The status word and the arrival counters must start at zero; a previous
  // call leaves the counters at zero, but one that stopped on a device-side
  // error may not. The partials are written before they are read.
  if (cudaMemsetAsync(scratch, 0, kCtrlBytes + (size_t)nst * 4, stream) != cudaSuccess) return DMS_ERR_CUDA;
  cudaError_t e = launch_attention(dv, plan, stream, n_seqs, seq_ids, Q, num_q_heads, scale, out,
                                   out_dtype == DMS_F32, AttnCounts{kv->retained, 0, 0},
                                   AttnGuess{nullptr, nullptr, false});
  return e == cudaSuccess ? DMS_OK : DMS_ERR_CUDA;
}

extern "C" dms_status dms_decode_attention_noalloc(cudaStream_t stream, const dms_paged_kv* kv, int32_t n_seqs,
                                                   const int32_t* seq_ids, const void* Q, int32_t num_q_heads,
                                                   float scale, void* out, dms_dtype out_dtype) {
  nvtxRangePushA("dms_decode_attention_noalloc");   // profiler timelines; a no-op without a tool
  const dms_status st = noalloc_impl(stream, kv, n_seqs, seq_ids, Q, num_q_heads, scale, out, out_dtype);
  nvtxRangePop();
  return st;
}
