// Query absorption and RoPE of the decoupled query, on CUDA cores (first version):
//   q_abs[b,i,0:512]   = W_UK,i^T q^C_{b,i}
//   q_abs[b,i,512:576] = RoPE_{kv_len[b]-1}(q^R_{b,i})
// One CTA per (head, 8 sequences); each thread owns two latent columns, so a W_UK row
// (512 bf16) is read as one coalesced 1 KB sweep per CTA.
#include "mla_internal.cuh"

namespace mla {
namespace {

constexpr int kThreads = 256;
constexpr int kBT = 8;  // sequences per CTA

__global__ void __launch_bounds__(kThreads)
absorb_q_simple(const __nv_bfloat16* __restrict__ q_c, const __nv_bfloat16* __restrict__ q_r,
                const __nv_bfloat16* __restrict__ w_uk, const int32_t* __restrict__ kv_lens,
                __nv_bfloat16* __restrict__ q_abs, int batch, int n_heads, double rope_base) {
  __shared__ float sq[kBT][kDHead];
  const int h = blockIdx.x, b0 = blockIdx.y * kBT, tid = threadIdx.x;
  for (int i = tid; i < kBT * kDHead; i += kThreads) {
    const int bb = i / kDHead, d = i % kDHead;
    const int b = b0 + bb;
    sq[bb][d] = b < batch ? __bfloat162float(q_c[((int64_t)b * n_heads + h) * kDHead + d]) : 0.f;
  }
  __syncthreads();

  float acc[kBT][2];
#pragma unroll
  for (int bb = 0; bb < kBT; ++bb) acc[bb][0] = acc[bb][1] = 0.f;
  const __nv_bfloat162* w = reinterpret_cast<const __nv_bfloat162*>(
      w_uk + (int64_t)h * kDHead * kDLatent) + tid;
#pragma unroll 4
  for (int d = 0; d < kDHead; ++d) {
    const float2 wv = __bfloat1622float2(w[d * (kDLatent / 2)]);
#pragma unroll
    for (int bb = 0; bb < kBT; ++bb) {
      acc[bb][0] = fmaf(sq[bb][d], wv.x, acc[bb][0]);
      acc[bb][1] = fmaf(sq[bb][d], wv.y, acc[bb][1]);
    }
  }
#pragma unroll
  for (int bb = 0; bb < kBT; ++bb) {
    const int b = b0 + bb;
    if (b < batch)
      reinterpret_cast<__nv_bfloat162*>(q_abs + ((int64_t)b * n_heads + h) * kRow)[tid] =
          __floats2bfloat162_rn(acc[bb][0], acc[bb][1]);
  }

  // RoPE: thread -> (sequence bb, pair m); angles in double (positions reach 2^17).
  {
    const int bb = tid / (kDRope / 2), m = tid % (kDRope / 2);
    const int b = b0 + bb;
    if (bb < kBT && b < batch) {
      const __nv_bfloat16* src = q_r + ((int64_t)b * n_heads + h) * kDRope + 2 * m;
      const double x0 = __bfloat162float(src[0]), x1 = __bfloat162float(src[1]);
      double y0 = x0, y1 = x1;
      if (rope_base != 0.0) {
        const int pos = max(kv_lens[b] - 1, 0);
        const double theta = pow(rope_base, -2.0 * m / kDRope);
        double sn, cs;
        sincos((double)pos * theta, &sn, &cs);
        y0 = x0 * cs - x1 * sn;
        y1 = x0 * sn + x1 * cs;
      }
      __nv_bfloat16* dst = q_abs + ((int64_t)b * n_heads + h) * kRow + kDLatent + 2 * m;
      dst[0] = __double2bfloat16(y0);
      dst[1] = __double2bfloat16(y1);
    }
  }
}

}  // namespace

cudaError_t launch_absorb_q(const mla_decode_s& h, int batch, const __nv_bfloat16* q_c,
                            const __nv_bfloat16* q_r, const __nv_bfloat16* w_uk,
                            const int32_t* kv_lens, __nv_bfloat16* q_abs, cudaStream_t s) {
  dim3 grid(h.cfg.n_heads, (batch + kBT - 1) / kBT);
  absorb_q_simple<<<grid, kThreads, 0, s>>>(q_c, q_r, w_uk, kv_lens, q_abs, batch,
                                            h.cfg.n_heads, (double)h.cfg.rope_base);
  return cudaGetLastError();
}

}  // namespace mla
