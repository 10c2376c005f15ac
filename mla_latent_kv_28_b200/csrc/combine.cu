// Log-sum-exp merge of the split partials of each (sequence, head):
//   lse* = max_s lse_s,  w_s = exp(lse_s - lse*),
//   latent = sum_s w_s O_s / sum_s w_s,  lse = lse* + log sum_s w_s.
// A sequence with no tokens gets latent 0 and lse -inf.
//
// The partials are stored [slot][column quad][head][4 floats] (the decode kernel's threads
// each own one head, so that layout makes its stores contiguous across a warp). A thread
// works on one head (so a warp's loads are contiguous 512-byte pieces) and QG column quads
// (its output is 8*QG contiguous bytes). Two shapes, picked on the host from how many
// splits a sequence can have:
//   few splits (QG = 4): a thread merges all of a sequence's slots for 16 columns;
//   many splits (QG = 1): the slots are dealt round-robin to SL threads per (head, quad),
//   which meet in shared memory for the max, the weights and the sums, so a single long
//   sequence split ~70 ways still has thousands of loads in flight.
#include <algorithm>
#include <type_traits>

#include "mla_internal.cuh"

namespace mla {
namespace {

constexpr int kThreads = 256;
constexpr int kQuads = kDLatent / 4;

// OutT: __nv_bfloat16 (the latent output) or float (the fp32 partial of a KV shard, merged
// later across GPUs).
template <int QG, typename OutT>
__global__ void __launch_bounds__(kThreads)
combine_kernel(PlanView plan, int n_heads, int slot_lanes, int groups_per_block,
               const float* __restrict__ part_o, const float* __restrict__ part_lse,
               OutT* __restrict__ out_latent, float* __restrict__ lse_out, int row_base, int out_rows) {
  // n_heads: the rows of the partials (one launch's group); out_rows: rows per sequence of the
  // outputs, of which this launch writes [row_base, row_base + n_heads)
  constexpr int kGroups = kQuads / QG;
  __shared__ float s_m[kThreads];
  __shared__ float4 s_acc[kThreads][QG];
  __shared__ float s_w[kThreads];
  const int blocks_per_seq = (kGroups + groups_per_block - 1) / groups_per_block;
  const int b = blockIdx.x / blocks_per_seq;
  const int tid = threadIdx.x, h = tid % n_heads, r = tid / n_heads;
  const int lanes = slot_lanes > 1 ? slot_lanes : groups_per_block;
  const bool active = tid < lanes * n_heads;
  const int sl = slot_lanes > 1 ? r : 0;
  const int grp = (blockIdx.x % blocks_per_seq) * groups_per_block + (slot_lanes > 1 ? 0 : r);
  grid_dependency_wait();   // the partials of the decode kernel
  allow_dependent_launch();
  const bool work = active && grp < kGroups;
  const int s0 = plan.seq_slot[b], s1 = plan.seq_slot[b + 1];
  const float* lse = part_lse + h;

  float m = -INFINITY;
  if (work) {
#pragma unroll 4
    for (int s = s0 + sl; s < s1; s += slot_lanes) m = fmaxf(m, lse[(int64_t)s * n_heads]);
  }
  if (slot_lanes > 1) {   // the max over all of the sequence's slots
    s_m[tid] = m;
    __syncthreads();
    for (int i = 0; i < slot_lanes; ++i) m = fmaxf(m, s_m[i * n_heads + h]);
  }
  float4 acc[QG];
#pragma unroll
  for (int q = 0; q < QG; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  if (work && m != -INFINITY) {
    const int64_t quad_stride = (int64_t)n_heads * 4;          // floats between quads
    const int64_t slot_stride = (int64_t)kQuads * quad_stride;  // floats between slots
    const float* o = part_o + (int64_t)grp * QG * quad_stride + h * 4;
#pragma unroll 4
    for (int s = s0 + sl; s < s1; s += slot_lanes) {
      const float w = __expf(lse[(int64_t)s * n_heads] - m);
      wsum += w;
#pragma unroll
      for (int q = 0; q < QG; ++q) {
        const float4 v = *reinterpret_cast<const float4*>(o + s * slot_stride + q * quad_stride);
        acc[q].x = fmaf(w, v.x, acc[q].x);
        acc[q].y = fmaf(w, v.y, acc[q].y);
        acc[q].z = fmaf(w, v.z, acc[q].z);
        acc[q].w = fmaf(w, v.w, acc[q].w);
      }
    }
  }
  if (slot_lanes > 1) {   // lane 0 of each (head, quad) adds the other lanes' sums
    __syncthreads();
#pragma unroll
    for (int q = 0; q < QG; ++q) s_acc[tid][q] = acc[q];
    s_w[tid] = wsum;
    __syncthreads();
    if (sl == 0) {
      for (int i = 1; i < slot_lanes; ++i) {
        const int t = i * n_heads + h;
        wsum += s_w[t];
#pragma unroll
        for (int q = 0; q < QG; ++q) {
          acc[q].x += s_acc[t][q].x; acc[q].y += s_acc[t][q].y;
          acc[q].z += s_acc[t][q].z; acc[q].w += s_acc[t][q].w;
        }
      }
    }
  }
  if (!work || sl != 0) return;
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  if constexpr (std::is_same<OutT, float>::value) {
    float* dst = out_latent + ((int64_t)b * out_rows + row_base + h) * kDLatent + grp * 4 * QG;
#pragma unroll
    for (int q = 0; q < QG; ++q)
      reinterpret_cast<float4*>(dst)[q] =
          make_float4(acc[q].x * inv, acc[q].y * inv, acc[q].z * inv, acc[q].w * inv);
    if (lse_out != nullptr && grp == 0)
      lse_out[(int64_t)b * out_rows + row_base + h] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
    return;
  }
  uint32_t packed[2 * QG];
#pragma unroll
  for (int q = 0; q < QG; ++q) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc[q].x * inv, acc[q].y * inv);
    __nv_bfloat162 hi = __floats2bfloat162_rn(acc[q].z * inv, acc[q].w * inv);
    packed[2 * q] = *reinterpret_cast<uint32_t*>(&lo);
    packed[2 * q + 1] = *reinterpret_cast<uint32_t*>(&hi);
  }
  __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(out_latent) + ((int64_t)b * out_rows + row_base + h) * kDLatent + grp * 4 * QG;
  if (QG == 4) {
    reinterpret_cast<uint4*>(dst)[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    reinterpret_cast<uint4*>(dst)[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
  } else {
#pragma unroll
    for (int q = 0; q < QG; ++q)
      reinterpret_cast<uint2*>(dst)[q] = make_uint2(packed[2 * q], packed[2 * q + 1]);
  }
  if (lse_out != nullptr && grp == 0)
    lse_out[(int64_t)b * out_rows + row_base + h] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
}

}  // namespace

template <typename OutT>
cudaError_t launch_combine_t(const mla_decode_s& h, int batch, OutT* out_latent, float* lse,
                             int row_base, cudaStream_t s) {
  const int n_heads = std::min(h.group_rows, h.n_rows - row_base);   // this group's rows
  const int per_block = n_heads >= kThreads ? 1 : kThreads / n_heads;   // head rows per block
  // the most slots one sequence can have: balanced units overlap about units / batch + 1 of a
  // sequence's tiles; capped plans give at most max_splits
  const int max_slots = h.cfg.max_splits > 0 ? h.cfg.max_splits : (h.units + batch - 1) / batch + 1;
  if (max_slots <= 4) {
    constexpr int kG = kQuads / 4;
    const int bps = (kG + per_block - 1) / per_block;
    return launch_pdl(combine_kernel<4, OutT>, dim3(batch * bps), dim3(kThreads), 0, s, h.ws.plan, n_heads,
                      1, per_block, (const float*)h.ws.part_o, (const float*)h.ws.part_lse,
                      out_latent, lse, row_base, h.n_rows);
  }
  return launch_pdl(combine_kernel<1, OutT>, dim3(batch * kQuads), dim3(kThreads), 0, s, h.ws.plan, n_heads,
                    per_block, 1, (const float*)h.ws.part_o, (const float*)h.ws.part_lse, out_latent,
                    lse, row_base, h.n_rows);
}

cudaError_t launch_combine(const mla_decode_s& h, int batch, __nv_bfloat16* out_latent,
                           float* lse, int row_base, cudaStream_t s) {
  return launch_combine_t(h, batch, out_latent, lse, row_base, s);
}

cudaError_t launch_combine_f32(const mla_decode_s& h, int batch, float* out_latent, float* lse,
                               int row_base, cudaStream_t s) {
  return launch_combine_t(h, batch, out_latent, lse, row_base, s);
}

}  // namespace mla
