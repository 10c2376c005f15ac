// The C ABI of libmla_decode.so: argument checks, the workspace, and the launches.
// Every compute call validates on the host, then enqueues kernels on the caller's stream;
// nothing here allocates after mla_decode_create.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>

#include "mla_internal.cuh"

namespace {

using mla::kDHead;
using mla::kDLatent;
using mla::kDRope;

constexpr int kCacheAlign = 16;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & (kCacheAlign - 1)) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int config_status(const mla_config_t* c) {
  if (c == nullptr) return MLA_ERR_INVALID_ARG;
  if (c->n_heads < 1 || c->max_batch < 1 || c->max_kv_len < 1 || c->max_splits < 0 ||
      c->page_size < 0 || !(c->softmax_scale >= 0.f) || !std::isfinite(c->softmax_scale) ||
      !(c->rope_base >= 0.f) || !std::isfinite(c->rope_base))
    return MLA_ERR_INVALID_ARG;
  if (c->d_head != kDHead || c->d_latent != kDLatent || c->d_rope != kDRope)
    return MLA_ERR_UNSUPPORTED;
  if (c->n_heads > mla::kMaxHeads || c->max_batch > mla::kMaxBatch) return MLA_ERR_UNSUPPORTED;
  if (c->page_size != 0 && c->page_size != 64) return MLA_ERR_UNSUPPORTED;
  if (c->max_kv_len > (int64_t)1 << 30) return MLA_ERR_UNSUPPORTED;
  if (c->max_splits > 64) return MLA_ERR_UNSUPPORTED;
  if (c->q_len < 0) return MLA_ERR_INVALID_ARG;
  {
    const int64_t T = c->q_len > 1 ? c->q_len : 1;
    if ((int64_t)c->n_heads * T > mla::kMaxRows || (int64_t)c->max_batch * T > mla::kMaxTokenRows)
      return MLA_ERR_UNSUPPORTED;
  }
  if (!(c->yarn_factor >= 0.f) || !std::isfinite(c->yarn_factor) ||
      (c->yarn_factor > 0.f && c->yarn_factor < 1.f))
    return MLA_ERR_INVALID_ARG;
  if (c->yarn_factor > 1.f &&
      (c->yarn_original_len < 1 || !std::isfinite(c->yarn_alpha) || !std::isfinite(c->yarn_beta) ||
       !(c->yarn_beta > c->yarn_alpha) || !(c->yarn_mscale_coef >= 0.f) ||
       !std::isfinite(c->yarn_mscale_coef)))
    return MLA_ERR_INVALID_ARG;
  return MLA_OK;
}

// Pair frequencies of the decoupled RoPE: base^(-2m/64), and with YaRN (factor s > 1) the
// blend of theta/s (pairs whose wavelength fits into the original context at most alpha
// times) and theta (at least beta times), linear in that count between the two.
void rope_frequencies(const mla_config_t& c, double* theta) {
  for (int m = 0; m < kDRope / 2; ++m) {
    if (!(c.rope_base > 0.f)) { theta[m] = 0.0; continue; }
    const double th = std::pow((double)c.rope_base, -2.0 * m / kDRope);
    if (!(c.yarn_factor > 1.f)) { theta[m] = th; continue; }
    const double fits = (double)c.yarn_original_len * th / (2.0 * 3.141592653589793);
    double w = (fits - (double)c.yarn_alpha) / ((double)c.yarn_beta - (double)c.yarn_alpha);
    w = std::min(1.0, std::max(0.0, w));
    theta[m] = w * th + (1.0 - w) * th / (double)c.yarn_factor;
  }
}

}  // namespace

extern "C" {

const char* mla_status_string(int status) {
  switch (status) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_OOM: return "MLA_ERR_OOM";
    case MLA_ERR_DEVICE_CHECK: return "MLA_ERR_DEVICE_CHECK";
    default: return "MLA_ERR_UNKNOWN";
  }
}

int mla_check_config(const mla_config_t* cfg) { return config_status(cfg); }

int mla_decode_create(const mla_config_t* cfg, int device, mla_handle_t* out) {
  if (out == nullptr) return MLA_ERR_INVALID_ARG;
  *out = nullptr;
  const int st = config_status(cfg);
  if (st != MLA_OK) return st;
  if (cudaSetDevice(device) != cudaSuccess) return MLA_ERR_CUDA;
  int major = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (major != 10) return MLA_ERR_UNSUPPORTED;  // built for sm_100a only

  mla_decode_s* h = new (std::nothrow) mla_decode_s;
  if (h == nullptr) return MLA_ERR_OOM;
  h->cfg = *cfg;
  h->device = device;
  h->num_sms = sms;
  double t = 1.0;   // YaRN's factor on the scores
  if (cfg->yarn_factor > 1.f) {
    const double root = (double)cfg->yarn_mscale_coef * std::log((double)cfg->yarn_factor) + 1.0;
    t = root * root;
  }
  h->scale = cfg->softmax_scale > 0.f ? cfg->softmax_scale
                                      : (float)(t / std::sqrt((double)(kDHead + kDRope)));
  rope_frequencies(*cfg, h->theta);
  h->q_len = cfg->q_len > 1 ? cfg->q_len : 1;
  h->n_rows = cfg->n_heads * h->q_len;
  h->group_rows = std::min(h->n_rows, mla::kMaxHeads);
  h->units = sms / 2;  // the decode kernel runs one 2-CTA cluster per unit of work

  const int B = cfg->max_batch;
  const int max_units = cfg->max_splits > 0 ? B * cfg->max_splits : h->units;
  const int max_slots = max_units + B;
  size_t off = 0;
  const size_t o_err = off;       off = round_up(off + 4, 256);
  const size_t o_hdr = off;       off = round_up(off + 4 * 4, 256);
  const size_t o_seq_tile = off;  off = round_up(off + 4 * (B + 1), 256);
  const size_t o_seq_slot = off;  off = round_up(off + 4 * (B + 1), 256);
  const size_t o_seq_len = off;   off = round_up(off + 4 * B, 256);
  const size_t o_seq_unit = off;  off = round_up(off + 4 * B, 256);
  const size_t o_ubegin = off;    off = round_up(off + 4 * (max_units + 1), 256);
  const size_t o_useq = off;      off = round_up(off + 4 * max_units, 256);
  const size_t o_plse = off;      off = round_up(off + 4 * (size_t)max_slots * h->group_rows, 256);
  const size_t o_po = off;        off = round_up(off + 4 * (size_t)max_slots * h->group_rows * kDLatent, 256);
  const size_t o_ap = off;        off = round_up(off + 4 * (size_t)mla::kAppendSlices * B * h->q_len * mla::kRow, 256);

  void* base = nullptr;
  if (cudaMalloc(&base, off) != cudaSuccess) {
    cudaGetLastError();
    delete h;
    return MLA_ERR_OOM;
  }
  if (cudaMemset(base, 0, off) != cudaSuccess) {
    cudaFree(base);
    delete h;
    return MLA_ERR_CUDA;
  }
  char* p = static_cast<char*>(base);
  h->ws.base = base;
  h->ws.bytes = off;
  h->ws.err = reinterpret_cast<uint32_t*>(p + o_err);
  h->ws.plan.header = reinterpret_cast<int32_t*>(p + o_hdr);
  h->ws.plan.seq_tile = reinterpret_cast<int32_t*>(p + o_seq_tile);
  h->ws.plan.seq_slot = reinterpret_cast<int32_t*>(p + o_seq_slot);
  h->ws.plan.seq_len = reinterpret_cast<int32_t*>(p + o_seq_len);
  h->ws.plan.seq_unit = reinterpret_cast<int32_t*>(p + o_seq_unit);
  h->ws.plan.unit_begin = reinterpret_cast<int32_t*>(p + o_ubegin);
  h->ws.plan.unit_seq = reinterpret_cast<int32_t*>(p + o_useq);
  h->ws.part_lse = reinterpret_cast<float*>(p + o_plse);
  h->ws.part_o = reinterpret_cast<float*>(p + o_po);
  h->ws.append_part = reinterpret_cast<float*>(p + o_ap);
  h->ws.max_units = max_units;
  h->ws.max_slots = max_slots;
  *out = h;
  return MLA_OK;
}

int mla_destroy(mla_handle_t h) {
  if (h == nullptr) return MLA_OK;
  int st = MLA_OK;
  if (cudaSetDevice(h->device) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess)
    st = MLA_ERR_CUDA;
  if (h->ws.base != nullptr && cudaFree(h->ws.base) != cudaSuccess) st = MLA_ERR_CUDA;
  delete h;
  return st;
}

int64_t mla_workspace_bytes(mla_handle_t h) { return h == nullptr ? -1 : (int64_t)h->ws.bytes; }

int mla_absorb_q(mla_handle_t h, int32_t batch, const void* q_c, const void* q_r,
                 const void* w_uk, const int32_t* kv_lens, void* q_abs, mla_stream_t stream) {
  if (h == nullptr || q_c == nullptr || q_r == nullptr || w_uk == nullptr ||
      kv_lens == nullptr || q_abs == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (batch < 1 || batch > h->cfg.max_batch) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_c) || !aligned16(q_r) || !aligned16(w_uk) || !aligned16(q_abs))
    return MLA_ERR_INVALID_ARG;
  // one GEMM row per (sequence, new token)
  const cudaError_t e = mla::launch_absorb_q(
      *h, batch * h->q_len, static_cast<const __nv_bfloat16*>(q_c), static_cast<const __nv_bfloat16*>(q_r),
      static_cast<const __nv_bfloat16*>(w_uk), kv_lens, static_cast<__nv_bfloat16*>(q_abs), stream);
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

namespace {

// The cache arguments of the attention calls, checked against the handle.
int cache_view(const mla_decode_s* h, const void* c_kv, const void* k_r, int64_t row_stride,
               int64_t seq_stride, const int32_t* page_table, int32_t max_pages, int32_t num_pages,
               mla::CacheView* cv) {
  if (!aligned16(c_kv) || !aligned16(k_r)) return MLA_ERR_INVALID_ARG;
  if (row_stride < kDLatent || row_stride % 8 != 0) return MLA_ERR_INVALID_ARG;
  *cv = mla::CacheView{};
  cv->c_kv = static_cast<const __nv_bfloat16*>(c_kv);
  cv->k_r = static_cast<const __nv_bfloat16*>(k_r);
  cv->row_stride = row_stride;
  cv->page_size = h->cfg.page_size;
  if (h->cfg.page_size == 0) {
    if (page_table != nullptr || seq_stride < h->cfg.max_kv_len) return MLA_ERR_INVALID_ARG;
    cv->seq_stride = seq_stride;
  } else {
    const int64_t need = (h->cfg.max_kv_len + h->cfg.page_size - 1) / h->cfg.page_size;
    if (page_table == nullptr || max_pages < need || num_pages < 1) return MLA_ERR_INVALID_ARG;
    cv->page_table = page_table;
    cv->max_pages = max_pages;
    cv->num_pages = num_pages;
  }
  return MLA_OK;
}

// The arguments of the attention calls, checked; the cache as a view.
int attention_args(mla_handle_t h, int32_t batch, const void* q_abs, const void* c_kv,
                   const void* k_r, int64_t row_stride, int64_t seq_stride, const int32_t* kv_lens,
                   const int32_t* page_table, int32_t max_pages, int32_t num_pages,
                   const void* out_latent, const float* lse, mla::CacheView* cv) {
  if (h == nullptr || q_abs == nullptr || c_kv == nullptr || k_r == nullptr ||
      kv_lens == nullptr || out_latent == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (batch < 1 || batch > h->cfg.max_batch) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_abs) || !aligned16(out_latent) ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3) != 0))
    return MLA_ERR_INVALID_ARG;
  return cache_view(h, c_kv, k_r, row_stride, seq_stride, page_table, max_pages, num_pages, cv);
}

// The shared body of mla_decode_attn (bf16 latent), mla_decode_attn_partial (fp32) and the
// fused step (plan_built: the absorption kernel has built the work plan already).
int decode_attn_common(mla_handle_t h, int32_t batch, const void* q_abs, const void* c_kv,
                       const void* k_r, int64_t row_stride, int64_t seq_stride,
                       const int32_t* kv_lens, const int32_t* page_table, int32_t max_pages,
                       int32_t num_pages, void* out_latent, bool out_f32, float* lse,
                       mla_stream_t stream, bool plan_built = false) {
  mla::CacheView cv{};
  const int st = attention_args(h, batch, q_abs, c_kv, k_r, row_stride, seq_stride, kv_lens,
                                page_table, max_pages, num_pages, out_latent, lse, &cv);
  if (st != MLA_OK) return st;
  cudaError_t e = plan_built ? cudaSuccess : mla::launch_split_plan(*h, batch, kv_lens, stream);
  // more than 128 attention rows per sequence (several new tokens): one decode + combine per
  // group of 128 rows, each over the same cache and plan
  for (int rb = 0; e == cudaSuccess && rb < h->n_rows; rb += h->group_rows) {
    e = mla::launch_decode_split(*h, batch, static_cast<const __nv_bfloat16*>(q_abs), cv, rb, stream);
    if (e == cudaSuccess)
      e = out_f32 ? mla::launch_combine_f32(*h, batch, static_cast<float*>(out_latent), lse, rb, stream)
                  : mla::launch_combine(*h, batch, static_cast<__nv_bfloat16*>(out_latent), lse, rb, stream);
  }
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace

int mla_prefill_attn(mla_handle_t h, int32_t batch, const void* q_abs, const void* c_kv,
                     const void* k_r, int64_t row_stride, int64_t seq_stride,
                     const int32_t* kv_lens, const int32_t* page_table, int32_t max_pages,
                     int32_t num_pages, void* out_latent, float* lse, mla_stream_t stream) {
  if (h == nullptr || q_abs == nullptr || c_kv == nullptr || k_r == nullptr ||
      kv_lens == nullptr || out_latent == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (batch < 1 || batch > h->cfg.max_batch) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_abs) || !aligned16(out_latent) ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3) != 0))
    return MLA_ERR_INVALID_ARG;
  mla::CacheView cv;
  const int st = cache_view(h, c_kv, k_r, row_stride, seq_stride, page_table, max_pages, num_pages, &cv);
  if (st != MLA_OK) return st;
  cv.kv_lens = kv_lens;
  const cudaError_t e = mla::launch_prefill(*h, batch, static_cast<const __nv_bfloat16*>(q_abs), cv,
                                            static_cast<__nv_bfloat16*>(out_latent), lse, stream);
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int mla_decode_attn(mla_handle_t h, int32_t batch, const void* q_abs, const void* c_kv,
                    const void* k_r, int64_t row_stride, int64_t seq_stride,
                    const int32_t* kv_lens, const int32_t* page_table, int32_t max_pages,
                    int32_t num_pages, void* out_latent, float* lse, mla_stream_t stream) {
  return decode_attn_common(h, batch, q_abs, c_kv, k_r, row_stride, seq_stride, kv_lens, page_table,
                            max_pages, num_pages, out_latent, false, lse, stream);
}

int mla_decode_attn_fp8(mla_handle_t h, int32_t batch, const void* q_abs, const void* kv_codes,
                        const int8_t* kv_exp, int64_t row_stride, int64_t seq_stride,
                        const int32_t* kv_lens, const int32_t* page_table, int32_t max_pages,
                        int32_t num_pages, void* out_latent, float* lse, mla_stream_t stream) {
  if (h == nullptr || q_abs == nullptr || kv_codes == nullptr || kv_exp == nullptr ||
      kv_lens == nullptr || out_latent == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (batch < 1 || batch > h->cfg.max_batch) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_abs) || !aligned16(kv_codes) || !aligned16(out_latent) ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3) != 0))
    return MLA_ERR_INVALID_ARG;
  if (row_stride < mla::kRow || row_stride % 16 != 0) return MLA_ERR_INVALID_ARG;   // bytes
  mla::CacheView cv{};
  cv.c_kv = static_cast<const __nv_bfloat16*>(kv_codes);   // read as bytes by the kernel
  cv.k_r = nullptr;
  cv.row_stride = row_stride;
  cv.page_size = h->cfg.page_size;
  cv.kv_exp = kv_exp;
  if (h->cfg.page_size == 0) {
    if (page_table != nullptr || seq_stride < h->cfg.max_kv_len) return MLA_ERR_INVALID_ARG;
    cv.seq_stride = seq_stride;
  } else {
    const int64_t need = (h->cfg.max_kv_len + h->cfg.page_size - 1) / h->cfg.page_size;
    if (page_table == nullptr || max_pages < need || num_pages < 1) return MLA_ERR_INVALID_ARG;
    cv.page_table = page_table;
    cv.max_pages = max_pages;
    cv.num_pages = num_pages;
  }
  cudaError_t e = mla::launch_split_plan(*h, batch, kv_lens, stream);
  for (int rb = 0; e == cudaSuccess && rb < h->n_rows; rb += h->group_rows) {
    e = mla::launch_decode_split(*h, batch, static_cast<const __nv_bfloat16*>(q_abs), cv, rb, stream);
    if (e == cudaSuccess)
      e = mla::launch_combine(*h, batch, static_cast<__nv_bfloat16*>(out_latent), lse, rb, stream);
  }
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int mla_decode_attn_partial(mla_handle_t h, int32_t batch, const void* q_abs, const void* c_kv,
                            const void* k_r, int64_t row_stride, int64_t seq_stride,
                            const int32_t* kv_lens, const int32_t* page_table, int32_t max_pages,
                            int32_t num_pages, float* out_latent, float* lse, mla_stream_t stream) {
  if (h == nullptr || lse == nullptr) return MLA_ERR_INVALID_ARG;
  // several new tokens attend causally by their global positions, which a shard's local row
  // count does not carry
  if (h->q_len > 1) return MLA_ERR_UNSUPPORTED;
  return decode_attn_common(h, batch, q_abs, c_kv, k_r, row_stride, seq_stride, kv_lens, page_table,
                            max_pages, num_pages, out_latent, true, lse, stream);
}

int mla_merge_partials(mla_handle_t h, int32_t batch, int32_t n_parts, const float* latent_parts,
                       const float* lse_parts, void* out_latent, float* lse, mla_stream_t stream) {
  if (h == nullptr || latent_parts == nullptr || lse_parts == nullptr || out_latent == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (batch < 1 || batch > h->cfg.max_batch || n_parts < 1) return MLA_ERR_INVALID_ARG;
  if (!aligned16(latent_parts) || !aligned16(out_latent) ||
      (reinterpret_cast<uintptr_t>(lse_parts) & 3) != 0 ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3) != 0))
    return MLA_ERR_INVALID_ARG;
  const cudaError_t e = mla::launch_merge_parts(*h, batch, n_parts, latent_parts, lse_parts,
                                                static_cast<__nv_bfloat16*>(out_latent), lse, stream);
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

namespace {

// The shared body of mla_append_kv (bf16 rows) and mla_append_kv_fp8 (kv_exp != nullptr:
// E4M3 codes at c_kv, row_stride in bytes).
int append_kv_common(mla_handle_t h, int32_t batch, int32_t d_model, const void* hidden,
                     const void* w_dkv, const void* w_kr, const void* gamma, float rms_eps,
                     void* c_kv, void* k_r, int8_t* kv_exp, int64_t row_stride, int64_t seq_stride,
                     const int32_t* kv_lens, const int32_t* page_table, int32_t max_pages,
                     int32_t num_pages, mla_stream_t stream) {
  if (h == nullptr || hidden == nullptr || w_dkv == nullptr || w_kr == nullptr ||
      gamma == nullptr || c_kv == nullptr || k_r == nullptr || kv_lens == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (batch < 1 || batch > h->cfg.max_batch) return MLA_ERR_INVALID_ARG;
  if (d_model < 64 || d_model % 64 != 0) return MLA_ERR_INVALID_ARG;
  if (d_model > 8192) return MLA_ERR_UNSUPPORTED;
  if (!(rms_eps >= 0.f) || !std::isfinite(rms_eps)) return MLA_ERR_INVALID_ARG;
  if (!aligned16(hidden) || !aligned16(w_dkv) || !aligned16(w_kr) || !aligned16(gamma) ||
      !aligned16(c_kv) || !aligned16(k_r))
    return MLA_ERR_INVALID_ARG;
  if (kv_exp == nullptr ? (row_stride < kDLatent || row_stride % 8 != 0)
                        : (row_stride < mla::kRow || row_stride % 16 != 0))
    return MLA_ERR_INVALID_ARG;
  mla::CacheView cv{};
  cv.c_kv = static_cast<const __nv_bfloat16*>(c_kv);
  cv.k_r = static_cast<const __nv_bfloat16*>(k_r);
  cv.row_stride = row_stride;
  cv.page_size = h->cfg.page_size;
  cv.kv_exp = kv_exp;
  if (h->cfg.page_size == 0) {
    if (page_table != nullptr || seq_stride < h->cfg.max_kv_len) return MLA_ERR_INVALID_ARG;
    cv.seq_stride = seq_stride;
  } else {
    const int64_t need = (h->cfg.max_kv_len + h->cfg.page_size - 1) / h->cfg.page_size;
    if (page_table == nullptr || max_pages < need || num_pages < 1) return MLA_ERR_INVALID_ARG;
    cv.page_table = page_table;
    cv.max_pages = max_pages;
    cv.num_pages = num_pages;
  }
  const cudaError_t e = mla::launch_append_kv(
      *h, batch, d_model, static_cast<const __nv_bfloat16*>(hidden),
      static_cast<const __nv_bfloat16*>(w_dkv), static_cast<const __nv_bfloat16*>(w_kr),
      static_cast<const __nv_bfloat16*>(gamma), rms_eps, cv, static_cast<__nv_bfloat16*>(c_kv),
      static_cast<__nv_bfloat16*>(k_r), kv_lens, stream);
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

}  // namespace

int mla_append_kv(mla_handle_t h, int32_t batch, int32_t d_model, const void* hidden,
                  const void* w_dkv, const void* w_kr, const void* gamma, float rms_eps,
                  void* c_kv, void* k_r, int64_t row_stride, int64_t seq_stride,
                  const int32_t* kv_lens, const int32_t* page_table, int32_t max_pages,
                  int32_t num_pages, mla_stream_t stream) {
  return append_kv_common(h, batch, d_model, hidden, w_dkv, w_kr, gamma, rms_eps, c_kv, k_r, nullptr,
                          row_stride, seq_stride, kv_lens, page_table, max_pages, num_pages, stream);
}

int mla_append_kv_fp8(mla_handle_t h, int32_t batch, int32_t d_model, const void* hidden,
                      const void* w_dkv, const void* w_kr, const void* gamma, float rms_eps,
                      void* kv_codes, int8_t* kv_exp, int64_t row_stride, int64_t seq_stride,
                      const int32_t* kv_lens, const int32_t* page_table, int32_t max_pages,
                      int32_t num_pages, mla_stream_t stream) {
  if (kv_exp == nullptr) return MLA_ERR_INVALID_ARG;
  return append_kv_common(h, batch, d_model, hidden, w_dkv, w_kr, gamma, rms_eps, kv_codes,
                          kv_codes, kv_exp, row_stride, seq_stride, kv_lens, page_table, max_pages,
                          num_pages, stream);
}

int mla_apply_wuv(mla_handle_t h, int32_t batch, const void* latent, const void* w_uv,
                  void* out, mla_stream_t stream) {
  if (h == nullptr || latent == nullptr || w_uv == nullptr || out == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (batch < 1 || batch > h->cfg.max_batch) return MLA_ERR_INVALID_ARG;
  if (!aligned16(latent) || !aligned16(w_uv) || !aligned16(out)) return MLA_ERR_INVALID_ARG;
  const cudaError_t e = mla::launch_apply_wuv(
      *h, batch * h->q_len, static_cast<const __nv_bfloat16*>(latent),
      static_cast<const __nv_bfloat16*>(w_uv), static_cast<__nv_bfloat16*>(out), stream);
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int mla_decode_step(mla_handle_t h, int32_t batch, const void* q_c, const void* q_r,
                    const void* w_uk, const void* w_uv, const void* c_kv, const void* k_r,
                    int64_t row_stride, int64_t seq_stride, const int32_t* kv_lens,
                    const int32_t* page_table, int32_t max_pages, int32_t num_pages, void* q_abs,
                    void* latent, void* out, mla_stream_t stream) {
  // every argument is checked before anything is launched
  if (h == nullptr || q_c == nullptr || q_r == nullptr || w_uk == nullptr || w_uv == nullptr ||
      out == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_c) || !aligned16(q_r) || !aligned16(w_uk) || !aligned16(w_uv) || !aligned16(out))
    return MLA_ERR_INVALID_ARG;
  mla::CacheView cv{};
  const int st = attention_args(h, batch, q_abs, c_kv, k_r, row_stride, seq_stride, kv_lens,
                                page_table, max_pages, num_pages, latent, nullptr, &cv);
  if (st != MLA_OK) return st;
  // the absorption, with the work plan built beside it; one GEMM row per (sequence, new token)
  cudaError_t e = mla::launch_absorb_q_with_plan(
      *h, batch * h->q_len, batch, static_cast<const __nv_bfloat16*>(q_c),
      static_cast<const __nv_bfloat16*>(q_r), static_cast<const __nv_bfloat16*>(w_uk), kv_lens,
      static_cast<__nv_bfloat16*>(q_abs), stream);
  if (e != cudaSuccess) return MLA_ERR_CUDA;
  const int st2 = decode_attn_common(h, batch, q_abs, c_kv, k_r, row_stride, seq_stride, kv_lens,
                                     page_table, max_pages, num_pages, latent, false, nullptr,
                                     stream, true);
  if (st2 != MLA_OK) return st2;
  e = mla::launch_apply_wuv(*h, batch * h->q_len, static_cast<const __nv_bfloat16*>(latent),
                            static_cast<const __nv_bfloat16*>(w_uv), static_cast<__nv_bfloat16*>(out),
                            stream);
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int mla_absorb_q_fp8(mla_handle_t h, int32_t batch, const void* q_c, const void* q_r,
                     const void* w_uk_codes, const int8_t* w_uk_exp, const int32_t* kv_lens,
                     void* q_abs, mla_stream_t stream) {
  if (h == nullptr || q_c == nullptr || q_r == nullptr || w_uk_codes == nullptr ||
      w_uk_exp == nullptr || kv_lens == nullptr || q_abs == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (batch < 1 || batch > h->cfg.max_batch) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_c) || !aligned16(q_r) || !aligned16(w_uk_codes) || !aligned16(q_abs))
    return MLA_ERR_INVALID_ARG;
  const cudaError_t e = mla::launch_absorb_q_fp8(
      *h, batch * h->q_len, static_cast<const __nv_bfloat16*>(q_c), static_cast<const __nv_bfloat16*>(q_r),
      static_cast<const uint8_t*>(w_uk_codes), w_uk_exp, kv_lens, static_cast<__nv_bfloat16*>(q_abs), stream);
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int mla_apply_wuv_fp8(mla_handle_t h, int32_t batch, const void* latent, const void* w_uv_codes,
                      const int8_t* w_uv_exp, void* out, mla_stream_t stream) {
  if (h == nullptr || latent == nullptr || w_uv_codes == nullptr || w_uv_exp == nullptr ||
      out == nullptr)
    return MLA_ERR_INVALID_ARG;
  if (batch < 1 || batch > h->cfg.max_batch) return MLA_ERR_INVALID_ARG;
  if (!aligned16(latent) || !aligned16(w_uv_codes) || !aligned16(out)) return MLA_ERR_INVALID_ARG;
  const cudaError_t e = mla::launch_apply_wuv_fp8(
      *h, batch * h->q_len, static_cast<const __nv_bfloat16*>(latent),
      static_cast<const uint8_t*>(w_uv_codes), w_uv_exp, static_cast<__nv_bfloat16*>(out), stream);
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

int mla_check_device_errors(mla_handle_t h, mla_stream_t stream, uint32_t* detail) {
  if (h == nullptr) return MLA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MLA_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, h->ws.err, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (detail != nullptr) *detail = word;
  if (word == 0) return MLA_OK;
  if (cudaMemset(h->ws.err, 0, sizeof(word)) != cudaSuccess) return MLA_ERR_CUDA;
  return MLA_ERR_DEVICE_CHECK;
}

}  // extern "C"
