// Log-sum-exp merge of attention partials computed over disjoint pieces of each sequence's
// cache, e.g. on the GPUs that each hold one contiguous shard of a long request's tokens:
//   lse* = max_p lse_p,  w_p = exp(lse_p - lse*),
//   latent = sum_p w_p latent_p / sum_p w_p,  lse = lse* + log sum_p w_p
// (the merge of the split combine, over parts that arrive already normalised). A row whose
// parts are all empty (lse -inf) gets latent 0 and lse -inf.
//
// Layout: latent_parts [n_parts][batch][rows][512] fp32, lse_parts [n_parts][batch][rows];
// one thread per (sequence, row, 4 latent columns), the parts summed in part order.
#include "mla_internal.cuh"

namespace mla {
namespace {

constexpr int kThreads = 256;
constexpr int kQuads = kDLatent / 4;   // 128 threads per row

__global__ void __launch_bounds__(kThreads)
merge_parts_kernel(int n_parts, int64_t n_rows_total, const float* __restrict__ latent_parts,
                   const float* __restrict__ lse_parts, __nv_bfloat16* __restrict__ out,
                   float* __restrict__ lse_out) {
  grid_dependency_wait();
  allow_dependent_launch();
  const int64_t row = (int64_t)blockIdx.x * (kThreads / kQuads) + threadIdx.x / kQuads;
  const int q = threadIdx.x % kQuads;
  if (row >= n_rows_total) return;
  float m = -INFINITY;
  for (int i = 0; i < n_parts; ++i) m = fmaxf(m, lse_parts[(int64_t)i * n_rows_total + row]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  if (m != -INFINITY) {
    for (int i = 0; i < n_parts; ++i) {
      const float w = __expf(lse_parts[(int64_t)i * n_rows_total + row] - m);
      const float4 v = reinterpret_cast<const float4*>(latent_parts + ((int64_t)i * n_rows_total + row) * kDLatent)[q];
      wsum += w;
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
  reinterpret_cast<uint2*>(out + row * kDLatent)[q] =
      make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
  if (lse_out != nullptr && q == 0) lse_out[row] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
}

}  // namespace

cudaError_t launch_merge_parts(const mla_decode_s& h, int batch, int n_parts, const float* latent_parts,
                               const float* lse_parts, __nv_bfloat16* out_latent, float* lse_out,
                               cudaStream_t s) {
  const int64_t rows = (int64_t)batch * h.n_rows;
  const int per_block = kThreads / kQuads;
  const int64_t blocks = (rows + per_block - 1) / per_block;
  return launch_pdl(merge_parts_kernel, dim3((unsigned)blocks), dim3(kThreads), 0, s, n_parts, rows,
                    latent_parts, lse_parts, out_latent, lse_out);
}

}  // namespace mla
