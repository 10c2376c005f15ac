// V up-projection on CUDA cores (first version): out[b,i,:] = W_UV,i latent[b,i,:].
// One CTA per (head, 8 sequences); a warp takes 16 output rows d and reads each W_UV row
// (512 bf16) as 32 lanes x 32 bytes, reducing the 8 dot products across the warp.
#include "mla_internal.cuh"

namespace mla {
namespace {

constexpr int kThreads = 256;
constexpr int kBT = 8;

__global__ void __launch_bounds__(kThreads)
apply_wuv_simple(const __nv_bfloat16* __restrict__ latent, const __nv_bfloat16* __restrict__ w_uv,
                 __nv_bfloat16* __restrict__ out, int batch, int n_heads) {
  __shared__ float sl[kBT][kDLatent];
  const int h = blockIdx.x, b0 = blockIdx.y * kBT;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < kBT * kDLatent; i += kThreads) {
    const int bb = i / kDLatent, c = i % kDLatent;
    const int b = b0 + bb;
    sl[bb][c] = b < batch ? __bfloat162float(latent[((int64_t)b * n_heads + h) * kDLatent + c]) : 0.f;
  }
  __syncthreads();
  for (int d = warp * (kDHead / 8); d < (warp + 1) * (kDHead / 8); ++d) {
    const uint4* wrow = reinterpret_cast<const uint4*>(w_uv + ((int64_t)h * kDHead + d) * kDLatent);
    float acc[kBT];
#pragma unroll
    for (int bb = 0; bb < kBT; ++bb) acc[bb] = 0.f;
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      const int piece = part * 32 + lane;  // 8 bf16 per piece, 64 pieces per row
      const uint4 raw = wrow[piece];
      const __nv_bfloat162* wv = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(wv[k]);
        const int c = piece * 8 + 2 * k;
#pragma unroll
        for (int bb = 0; bb < kBT; ++bb)
          acc[bb] = fmaf(f.x, sl[bb][c], fmaf(f.y, sl[bb][c + 1], acc[bb]));
      }
    }
#pragma unroll
    for (int bb = 0; bb < kBT; ++bb)
      for (int o = 16; o; o >>= 1) acc[bb] += __shfl_xor_sync(0xffffffffu, acc[bb], o);
    if (lane < kBT) {
      const int b = b0 + lane;
      float v = 0.f;
#pragma unroll
      for (int bb = 0; bb < kBT; ++bb) v = (bb == lane) ? acc[bb] : v;
      if (b < batch) out[((int64_t)b * n_heads + h) * kDHead + d] = __float2bfloat16(v);
    }
  }
}

}  // namespace

cudaError_t launch_apply_wuv(const mla_decode_s& h, int batch, const __nv_bfloat16* latent,
                             const __nv_bfloat16* w_uv, __nv_bfloat16* out, cudaStream_t s) {
  dim3 grid(h.cfg.n_heads, (batch + kBT - 1) / kBT);
  apply_wuv_simple<<<grid, kThreads, 0, s>>>(latent, w_uv, out, batch, h.cfg.n_heads);
  return cudaGetLastError();
}

}  // namespace mla
