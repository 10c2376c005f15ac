// mla_decode_attn_noalloc: the split-KV decode attention for callers that cannot allocate
// device memory.
//
// Who needs it: a serving engine that has already reserved nearly all of HBM for its own
// KV-cache page pool and hands memory out only through that pool; a plugin hosted by a
// framework whose memory manager owns the device and forbids direct cudaMalloc; code on a
// latency-critical path where cudaMalloc / cudaFree (which may synchronise the device) are
// not acceptable. Such callers cannot create a handle, because mla_decode_create allocates
// the workspace. This entry point takes the configuration as arguments instead and keeps
// its scratch (work plan, split partials, error word) in one fixed-size array in device
// memory that is part of the library image.
//
// Costs and rules that follow from that:
//   * every GPU that loads the library holds the array (kScratchBytes) until the process
//     exits;
//   * all calls on a device share the one array, so calls whose kernels overlap on the GPU
//     (two streams, or two host threads) race and corrupt each other's partials; serialise
//     them;
//   * the array keeps the previous call's contents; each call clears the error word and
//     rewrites everything else it reads;
//   * the first call on a device looks up the array's device address (cudaGetSymbolAddress)
//     and caches it; make that first call before any stream capture. Only a successful
//     look-up is cached: if it fails (for instance inside a capture, or with an unrelated
//     error pending on the device), the call returns MLA_ERR_CUDA and the next call tries
//     again.
// The kernels are the same ones mla_decode_attn runs; only the scratch comes from here.
#include <algorithm>
#include <cmath>
#include <mutex>

#include "mla_internal.cuh"

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;   // 32 MiB per device
constexpr size_t kPlanBytes = size_t(64) << 10;      // error word + work plan region
constexpr int kNoAllocMaxBatch = 64;
constexpr int kMaxDevices = 64;

// The scratch. Host code must not use this name as a pointer: on the host it is only a
// stand-in for the symbol; its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

struct DeviceScratch {
  bool ready = false;             // the look-up below succeeded on this device
  unsigned char* base = nullptr;  // device address of g_scratch on this device
  int num_sms = 0;
  int major = 0;
};
DeviceScratch g_dev[kMaxDevices];
std::mutex g_dev_mutex;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// With the device current: find the array and the SM count, once per device. A failed
// look-up is not remembered, so a later call retries it.
cudaError_t device_scratch(int device, DeviceScratch* out) {
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  DeviceScratch& d = g_dev[device];
  if (!d.ready) {
    DeviceScratch n;
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n.num_sms, cudaDevAttrMultiProcessorCount, device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n.major, cudaDevAttrComputeCapabilityMajor, device);
    if (e != cudaSuccess) {
      cudaGetLastError();   // leave no error of the failed look-up behind for later calls
      return e;
    }
    n.base = static_cast<unsigned char*>(p);
    n.ready = true;
    d = n;
  }
  *out = d;
  return cudaSuccess;
}

}  // namespace

extern "C" int mla_decode_attn_noalloc(int32_t n_heads, float softmax_scale, int32_t page_size,
                                       int64_t max_kv_len, int32_t batch, const void* q_abs,
                                       const void* c_kv, const void* k_r, int64_t row_stride,
                                       int64_t seq_stride, const int32_t* kv_lens,
                                       const int32_t* page_table, int32_t max_pages,
                                       int32_t num_pages, void* out_latent, float* lse,
                                       uint32_t* err_word, mla_stream_t stream) {
  using namespace mla;
  // ---- arguments (the same rules as mla_decode_attn, plus the scratch limits)
  if (q_abs == nullptr || c_kv == nullptr || k_r == nullptr || kv_lens == nullptr ||
      out_latent == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (n_heads < 1 || batch < 1 || max_kv_len < 1 || !(softmax_scale >= 0.f) ||
      !std::isfinite(softmax_scale))
    return MLA_ERR_INVALID_ARG;
  if (n_heads > kMaxHeads || batch > kNoAllocMaxBatch || max_kv_len > (int64_t(1) << 30))
    return MLA_ERR_UNSUPPORTED;
  if (page_size != 0 && page_size != 64) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(q_abs) || !aligned16(c_kv) || !aligned16(k_r) || !aligned16(out_latent) ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3) != 0) ||
      (err_word != nullptr && (reinterpret_cast<uintptr_t>(err_word) & 3) != 0))
    return MLA_ERR_INVALID_ARG;
  if (row_stride < kDLatent || row_stride % 8 != 0) return MLA_ERR_INVALID_ARG;
  CacheView cv{};
  cv.c_kv = static_cast<const __nv_bfloat16*>(c_kv);
  cv.k_r = static_cast<const __nv_bfloat16*>(k_r);
  cv.row_stride = row_stride;
  cv.page_size = page_size;
  if (page_size == 0) {
    if (page_table != nullptr || seq_stride < max_kv_len) return MLA_ERR_INVALID_ARG;
    cv.seq_stride = seq_stride;
  } else {
    if (page_table == nullptr || max_pages < (max_kv_len + page_size - 1) / page_size ||
        num_pages < 1)
      return MLA_ERR_INVALID_ARG;
    cv.page_table = page_table;
    cv.max_pages = max_pages;
    cv.num_pages = num_pages;
  }

  // ---- the device's scratch (looked up once per device)
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return MLA_ERR_CUDA;
  if (device < 0 || device >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  DeviceScratch ds;
  if (device_scratch(device, &ds) != cudaSuccess) return MLA_ERR_CUDA;
  const DeviceScratch* d = &ds;
  if (d->major != 10) return MLA_ERR_UNSUPPORTED;

  // ---- carve the scratch: plan region first, then the split partials. Fewer heads leave
  // room for more slots; the number of units is what fits after one slot per sequence.
  const size_t slot_bytes = size_t(n_heads) * (kDLatent + 1) * sizeof(float);
  const int max_slots = int((kScratchBytes - kPlanBytes - 1024) / slot_bytes);
  // one unit per 2-CTA cluster of the decode kernel, as the handle path plans it
  const int units = std::min(d->num_sms / 2, max_slots - batch);
  if (units < 1) return MLA_ERR_UNSUPPORTED;

  mla_decode_s h{};  // a handle on the stack: no allocation, scratch pointers into g_scratch
  h.cfg = mla_config_t{};
  h.cfg.n_heads = n_heads;
  h.q_len = 1;
  h.n_rows = n_heads;
  h.group_rows = n_heads;
  h.cfg.d_head = kDHead;
  h.cfg.d_latent = kDLatent;
  h.cfg.d_rope = kDRope;
  h.cfg.page_size = page_size;
  h.cfg.max_batch = batch;
  h.cfg.max_kv_len = max_kv_len;
  h.cfg.softmax_scale = softmax_scale;
  h.cfg.rope_base = 0.f;
  h.cfg.max_splits = 0;
  h.device = device;
  h.num_sms = d->num_sms;
  h.scale = softmax_scale > 0.f ? softmax_scale
                                : (float)(1.0 / std::sqrt((double)(kDHead + kDRope)));
  h.units = units;

  unsigned char* p = d->base;
  size_t off = 0;
  auto take = [&](size_t bytes) { unsigned char* q = p + off; off = round_up(off + bytes, 256); return q; };
  uint32_t* scratch_err = reinterpret_cast<uint32_t*>(take(4));
  h.ws.plan.header = reinterpret_cast<int32_t*>(take(16));
  h.ws.plan.seq_tile = reinterpret_cast<int32_t*>(take(4 * (batch + 1)));
  h.ws.plan.seq_slot = reinterpret_cast<int32_t*>(take(4 * (batch + 1)));
  h.ws.plan.seq_len = reinterpret_cast<int32_t*>(take(4 * batch));
  h.ws.plan.seq_unit = reinterpret_cast<int32_t*>(take(4 * batch));
  h.ws.plan.unit_begin = reinterpret_cast<int32_t*>(take(4 * (units + 1)));
  h.ws.plan.unit_seq = reinterpret_cast<int32_t*>(take(4 * units));
  if (off > kPlanBytes) return MLA_ERR_UNSUPPORTED;
  off = kPlanBytes;
  h.ws.part_lse = reinterpret_cast<float*>(take(sizeof(float) * size_t(units + batch) * n_heads));
  h.ws.part_o = reinterpret_cast<float*>(take(slot_bytes / (kDLatent + 1) * kDLatent * (units + batch)));
  if (off > kScratchBytes) return MLA_ERR_UNSUPPORTED;
  h.ws.base = d->base;
  h.ws.bytes = kScratchBytes;
  h.ws.max_units = units;
  h.ws.max_slots = units + batch;
  h.ws.err = err_word != nullptr ? err_word : scratch_err;

  // ---- the error word starts at zero; every other scratch byte read is written first
  if (cudaMemsetAsync(h.ws.err, 0, sizeof(uint32_t), stream) != cudaSuccess) return MLA_ERR_CUDA;
  cudaError_t e = launch_split_plan(h, batch, kv_lens, stream);
  if (e == cudaSuccess)
    e = launch_decode_split(h, batch, static_cast<const __nv_bfloat16*>(q_abs), cv, 0, stream);
  if (e == cudaSuccess)
    e = launch_combine(h, batch, static_cast<__nv_bfloat16*>(out_latent), lse, 0, stream);
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}
