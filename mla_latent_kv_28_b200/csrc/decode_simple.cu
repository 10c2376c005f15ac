// Split-KV decode attention on CUDA cores: the first, plain version of the decode kernel.
// One CTA per (unit, group of 16 heads); each segment of a unit (one sequence's tokens in
// that unit) produces a partial latent output and its log-sum-exp in a slot.
//
//   s_j = scale * q_abs . [c_j ; k^R_j],  running max / sum (online softmax),
//   O = sum_j exp(s_j - m) c_j,  partial = O / l,  lse = m + log l.
#include "mla_internal.cuh"

namespace mla {
namespace {

constexpr int kHG = 16;      // heads per CTA
constexpr int kChunk = 16;   // tokens staged in shared memory at a time
constexpr int kThreads = 256;

__device__ __forceinline__ const __nv_bfloat16* row_ptr(const __nv_bfloat16* base,
                                                        int64_t row, int64_t stride) {
  return base + row * stride;
}

// Row index of token j of sequence b, or -1 if its page-table entry is out of range.
__device__ __forceinline__ int64_t token_row(const CacheView& cv, int b, int j, uint32_t* err) {
  if (cv.page_table == nullptr) return (int64_t)b * cv.seq_stride + j;
  const int32_t page = cv.page_table[(int64_t)b * cv.max_pages + j / cv.page_size];
  if (page < 0 || page >= cv.num_pages) {
    atomicOr(err, kErrBadPage);
    return -1;
  }
  return (int64_t)page * cv.page_size + (j % cv.page_size);
}

__global__ void __launch_bounds__(kThreads)
decode_split_simple(const __nv_bfloat16* __restrict__ q_abs, CacheView cv, PlanView plan,
                    int batch, int n_heads, float scale_log2, float* __restrict__ part_o,
                    float* __restrict__ part_lse, uint32_t* err) {
  __shared__ __nv_bfloat16 sq[kHG][kRow];
  __shared__ __align__(16) __nv_bfloat16 skv[kChunk][kRow];
  __shared__ float sp[kHG][kChunk];
  __shared__ float s_alpha[kHG];
  __shared__ float s_m[kHG], s_l[kHG];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h0 = blockIdx.y * kHG;
  const int n_units = plan.header[1];

  for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
    const int ub = plan.unit_begin[u], ue = plan.unit_begin[u + 1];
    for (int b = plan.unit_seq[u]; b < batch && plan.seq_tile[b] < ue; ++b) {
      const int tb = plan.seq_tile[b], te = plan.seq_tile[b + 1];
      if (te <= ub) continue;
      const int L = plan.seq_len[b];
      const int j0 = (max(ub, tb) - tb) * kTileTokens;
      const int j1 = min((min(ue, te) - tb) * kTileTokens, L);
      const int slot = plan.seq_slot[b] + (u - plan.seq_unit[b]);

      __syncthreads();
      for (int i = tid; i < kHG * kRow; i += kThreads) {
        const int hh = i / kRow, k = i % kRow;
        const int h = h0 + hh;
        sq[hh][k] = h < n_heads ? q_abs[((int64_t)b * n_heads + h) * kRow + k]
                                : __float2bfloat16(0.f);
      }
      if (tid < kHG) { s_m[tid] = -INFINITY; s_l[tid] = 0.f; }
      float acc[kHG][2];
#pragma unroll
      for (int hh = 0; hh < kHG; ++hh) acc[hh][0] = acc[hh][1] = 0.f;

      for (int j = j0; j < j1; j += kChunk) {
        const int nj = min(kChunk, j1 - j);
        __syncthreads();
        // stage the rows (16-byte pieces: 64 c^KV pieces + 8 k^R pieces per row)
        for (int i = tid; i < kChunk * (kRow / 8); i += kThreads) {
          const int t = i / (kRow / 8), piece = i % (kRow / 8);
          uint4 v = make_uint4(0, 0, 0, 0);
          if (t < nj) {
            const int64_t r = token_row(cv, b, j + t, err);
            if (r >= 0) {
              const __nv_bfloat16* src = piece < kDLatent / 8
                  ? row_ptr(cv.c_kv, r, cv.row_stride) + piece * 8
                  : row_ptr(cv.k_r, r, cv.row_stride) + (piece - kDLatent / 8) * 8;
              v = *reinterpret_cast<const uint4*>(src);
            }
          }
          *reinterpret_cast<uint4*>(&skv[t][piece * 8]) = v;
        }
        __syncthreads();
        // scores, in the log2 domain
        for (int i = tid; i < kHG * kChunk; i += kThreads) {
          const int hh = i / kChunk, t = i % kChunk;
          float s = -INFINITY;
          if (t < nj && h0 + hh < n_heads) {
            float a = 0.f;
            for (int k = 0; k < kRow; ++k)
              a = fmaf(__bfloat162float(sq[hh][k]), __bfloat162float(skv[t][k]), a);
            s = a * scale_log2;
          }
          sp[hh][t] = s;
        }
        __syncthreads();
        // online softmax: warp w updates heads 2w and 2w+1
        for (int hh = warp * 2; hh < warp * 2 + 2; ++hh) {
          const float s = lane < kChunk ? sp[hh][lane] : -INFINITY;
          float mx = s;
          for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          const float m_old = s_m[hh];
          const float m_new = fmaxf(m_old, mx);
          float p = 0.f, alpha = 1.f;
          if (m_new != -INFINITY) {
            p = exp2f(s - m_new);
            alpha = exp2f(m_old - m_new);
          }
          float sum = p;
          for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
          if (lane < kChunk) sp[hh][lane] = p;
          __syncwarp();
          if (lane == 0) {
            s_alpha[hh] = alpha;
            s_m[hh] = m_new;
            s_l[hh] = s_l[hh] * alpha + sum;
          }
        }
        __syncthreads();
        // O = alpha * O + P V   (this thread: latent columns tid and tid + 256)
#pragma unroll
        for (int hh = 0; hh < kHG; ++hh) {
          const float al = s_alpha[hh];
          float a0 = acc[hh][0] * al, a1 = acc[hh][1] * al;
          for (int t = 0; t < nj; ++t) {
            const float p = sp[hh][t];
            a0 = fmaf(p, __bfloat162float(skv[t][tid]), a0);
            a1 = fmaf(p, __bfloat162float(skv[t][tid + 256]), a1);
          }
          acc[hh][0] = a0;
          acc[hh][1] = a1;
        }
      }
      __syncthreads();
      // partial result: normalised latent and its lse (natural log)
#pragma unroll
      for (int hh = 0; hh < kHG; ++hh) {
        const int h = h0 + hh;
        if (h >= n_heads) continue;
        const float l = s_l[hh];
        const float inv = l > 0.f ? 1.f / l : 0.f;
        float* dst = part_o + ((int64_t)slot * n_heads + h) * kDLatent;
        dst[tid] = acc[hh][0] * inv;
        dst[tid + 256] = acc[hh][1] * inv;
        if (tid == 0)
          part_lse[(int64_t)slot * n_heads + h] =
              l > 0.f ? (s_m[hh] + log2f(l)) * 0.69314718055994531f : -INFINITY;
      }
    }
  }
}

}  // namespace

cudaError_t launch_decode_split(const mla_decode_s& h, int batch, const __nv_bfloat16* q_abs,
                                const CacheView& cache, cudaStream_t s) {
  const int groups = (h.cfg.n_heads + kHG - 1) / kHG;
  const int max_units = h.cfg.max_splits == 0 ? h.units : batch * h.cfg.max_splits;
  dim3 grid(max_units, groups);
  decode_split_simple<<<grid, kThreads, 0, s>>>(q_abs, cache, h.ws.plan, batch, h.cfg.n_heads,
                                                h.scale * 1.4426950408889634f, h.ws.part_o,
                                                h.ws.part_lse, h.ws.err);
  return cudaGetLastError();
}

}  // namespace mla
