// Log-sum-exp merge of the split partials of each (sequence, head):
//   lse* = max_s lse_s,  w_s = exp(lse_s - lse*),
//   latent = sum_s w_s O_s / sum_s w_s,  lse = lse* + log sum_s w_s.
// A sequence with no tokens gets latent 0 and lse -inf.
#include "mla_internal.cuh"

namespace mla {
namespace {

constexpr int kThreads = 128;  // 4 latent columns per thread

__global__ void __launch_bounds__(kThreads)
combine_kernel(PlanView plan, int n_heads, const float* __restrict__ part_o,
               const float* __restrict__ part_lse, __nv_bfloat16* __restrict__ out_latent,
               float* __restrict__ lse_out) {
  const int b = blockIdx.x / n_heads, h = blockIdx.x % n_heads;
  const int s0 = plan.seq_slot[b], s1 = plan.seq_slot[b + 1];
  float m = -INFINITY;
  for (int s = s0; s < s1; ++s) m = fmaxf(m, part_lse[(int64_t)s * n_heads + h]);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  float wsum = 0.f;
  if (m != -INFINITY) {
    for (int s = s0; s < s1; ++s) {
      const float w = __expf(part_lse[(int64_t)s * n_heads + h] - m);
      wsum += w;
      const float4 o = *reinterpret_cast<const float4*>(
          part_o + ((int64_t)s * n_heads + h) * kDLatent + threadIdx.x * 4);
      acc[0] = fmaf(w, o.x, acc[0]);
      acc[1] = fmaf(w, o.y, acc[1]);
      acc[2] = fmaf(w, o.z, acc[2]);
      acc[3] = fmaf(w, o.w, acc[3]);
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat162 lo = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
  __nv_bfloat162 hi = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
  __nv_bfloat16* dst = out_latent + ((int64_t)b * n_heads + h) * kDLatent + threadIdx.x * 4;
  uint2 packed;
  packed.x = *reinterpret_cast<uint32_t*>(&lo);
  packed.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(dst) = packed;
  if (lse_out != nullptr && threadIdx.x == 0)
    lse_out[(int64_t)b * n_heads + h] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
}

}  // namespace

cudaError_t launch_combine(const mla_decode_s& h, int batch, __nv_bfloat16* out_latent,
                           float* lse, cudaStream_t s) {
  combine_kernel<<<batch * h.cfg.n_heads, kThreads, 0, s>>>(
      h.ws.plan, h.cfg.n_heads, h.ws.part_o, h.ws.part_lse, out_latent, lse);
  return cudaGetLastError();
}

}  // namespace mla
