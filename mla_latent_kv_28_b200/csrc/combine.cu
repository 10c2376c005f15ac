// Log-sum-exp merge of the split partials of each (sequence, head):
//   lse* = max_s lse_s,  w_s = exp(lse_s - lse*),
//   latent = sum_s w_s O_s / sum_s w_s,  lse = lse* + log sum_s w_s.
// A sequence with no tokens gets latent 0 and lse -inf.
//
// The partials are stored [slot][column quad][head][4 floats] (the decode kernel's threads
// each own one head, so that layout makes its stores contiguous across a warp). One thread
// merges one (sequence, column quad, head): a warp reads 32 heads' quads of a slot as one
// contiguous 512-byte piece. A sequence is cut into many small blocks, and the loop over its
// slots is unrolled, so even a batch of a few long sequences split many ways keeps enough
// loads in flight.
#include "mla_internal.cuh"

namespace mla {
namespace {

constexpr int kThreads = 256;
constexpr int kQuads = kDLatent / 4;

__global__ void __launch_bounds__(kThreads)
combine_kernel(PlanView plan, int n_heads, int quads_per_block, const float* __restrict__ part_o,
               const float* __restrict__ part_lse, __nv_bfloat16* __restrict__ out_latent,
               float* __restrict__ lse_out) {
  const int blocks_per_seq = (kQuads + quads_per_block - 1) / quads_per_block;
  const int b = blockIdx.x / blocks_per_seq;
  const int quad = (blockIdx.x % blocks_per_seq) * quads_per_block + threadIdx.x / n_heads;
  const int h = threadIdx.x % n_heads;
  grid_dependency_wait();   // the partials of the decode kernel
  allow_dependent_launch();
  if (threadIdx.x >= quads_per_block * n_heads || quad >= kQuads) return;
  const int s0 = plan.seq_slot[b], s1 = plan.seq_slot[b + 1];
  const float* lse = part_lse + h;

  float m = -INFINITY;
#pragma unroll 4
  for (int s = s0; s < s1; ++s) m = fmaxf(m, lse[(int64_t)s * n_heads]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  if (m != -INFINITY) {
    const float* o = part_o + ((int64_t)quad * n_heads + h) * 4;
    const int64_t slot_stride = (int64_t)kQuads * n_heads * 4;
#pragma unroll 4
    for (int s = s0; s < s1; ++s) {
      const float w = __expf(lse[(int64_t)s * n_heads] - m);
      const float4 v = *reinterpret_cast<const float4*>(o + s * slot_stride);
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
  uint2 packed;
  packed.x = *reinterpret_cast<uint32_t*>(&lo);
  packed.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(out_latent + ((int64_t)b * n_heads + h) * kDLatent + 4 * quad) = packed;
  if (lse_out != nullptr && quad == 0)
    lse_out[(int64_t)b * n_heads + h] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
}

}  // namespace

cudaError_t launch_combine(const mla_decode_s& h, int batch, __nv_bfloat16* out_latent,
                           float* lse, cudaStream_t s) {
  const int n_heads = h.cfg.n_heads;
  const int qpb = n_heads >= kThreads ? 1 : kThreads / n_heads;   // column quads per block
  const int blocks_per_seq = (kQuads + qpb - 1) / qpb;
  return launch_pdl(combine_kernel, dim3(batch * blocks_per_seq), dim3(kThreads), 0, s, h.ws.plan,
                    n_heads, qpb, (const float*)h.ws.part_o, (const float*)h.ws.part_lse,
                    out_latent, lse);
}

}  // namespace mla
