// The cache write of a decode step's new token, on the sm_100a tensor core:
//
//   x   = [W_DKV ; W_KR] h_b                              576 features, fp32 accumulation
//   row = [ RMSNorm(x[0:512]) * gamma ; RoPE_{kv_len-1}(x[512:576]) ]      bf16
//
// written as row kv_len[b]-1 of sequence b, in the cache layout the decode kernel reads
// (DeepSeek-V2 architecture page eq. 9 c^KV = W^DKV h; the paper notes' RMSNorm after the
// compressed latent; DeepSeek-V3 walkthrough section 2.2 k^R = RoPE(W^KR h), the two parts
// that are cached). With q_len new tokens per sequence, h is [B, q_len, d] and token t's row
// is kv_len[b] - q_len + t, rotated at that position. A quantised cache gets the row as E4M3
// codes with the smallest power-of-two scale that fits (its exponent stored beside).
//
// Kernel 1, kv_down_tc: the projection is bound by reading the weights (576 x d bf16, 5.9 MB
// at d = 5120), so it is cut into many CTAs: one per (128-feature block, slice of d, batch
// chunk). The weights are the M = 128 operand (four blocks of W_DKV, one of W_KR whose rows
// past 64 read as zero), the hidden states the N operand; four warps issue a quarter of the
// slice's K steps each into their own accumulator, and the slice's partial sums go to the
// handle's workspace. Kernel 2, kv_finalize: one CTA per (sequence, new token) row adds the
// slices' partials in a fixed order (so the result does not depend on timing), applies the
// RMSNorm and the rotation, and writes the row (bf16, or quantised).
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "mla_internal.cuh"
#include "sm100.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kThreads = 256;
constexpr int kIssuers = 4;
constexpr int kFeatBlocks = 5;                 // 576 features in 128-row blocks
constexpr uint32_t kWBox = 128 * 128;          // 128 rows x 64 columns bf16 = 16 KB

struct DownParams {
  int batch, n_tile, slice;      // slice: columns of d per CTA (a multiple of 64)
  uint32_t idesc;
  float* part;                   // [kAppendSlices][part_batch][576] fp32
  int part_batch;
  uint32_t* err;
  long long wait_limit;
};

__device__ __forceinline__ bool wait_landed(uint32_t bar, const DownParams& p) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, 0)) {
    if (clock64() - t0 > p.wait_limit) {
      atomicOr(p.err, kErrTimeout);
      return false;
    }
  }
  return true;
}

__global__ void __launch_bounds__(kThreads, 1)
kv_down_tc(const __grid_constant__ CUtensorMap tmap_wd, const __grid_constant__ CUtensorMap tmap_wr,
           const __grid_constant__ CUtensorMap tmap_h, const DownParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int nbox = p.slice / 64;                     // 64-column boxes of the slice
  const uint32_t hbox = (uint32_t)p.n_tile * 128;    // bytes of one hidden-state box
  const uint32_t hbase = sbase + nbox * kWBox;
  const uint32_t bars = hbase + nbox * hbox;          // [0] landed, [1..4] issuer q done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + (bars - sbase) + 8 * (1 + kIssuers));
  volatile int* ok_flags = reinterpret_cast<volatile int*>(smem + (bars - sbase) + 8 * (1 + kIssuers) + 4);
  const int mb = blockIdx.x, kc = blockIdx.y, b0 = blockIdx.z * p.n_tile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t col_stride = p.n_tile < 32 ? 32u : (uint32_t)p.n_tile;
  const uint32_t need = kIssuers * col_stride;
  const uint32_t tmem_cols = need <= 128 ? 128 : need <= 256 ? 256 : 512;
  const int x0 = kc * p.slice;                        // first column of d in this slice

  if (threadIdx.x == 0) {
    mbar_init(bars, 1);
    for (int q = 0; q < kIssuers; ++q) mbar_init(bars + 8 * (1 + q), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(mb < 4 ? &tmap_wd : &tmap_wr);
    prefetch_tmap(&tmap_h);
    // this CTA's weights into L2 while the previous kernel finishes (a hint only)
    for (int i = 0; i < nbox; ++i) tma_prefetch_2d(mb < 4 ? &tmap_wd : &tmap_wr, x0 + 64 * i, mb < 4 ? 128 * mb : 0);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dependency_wait();   // the hidden states may come from the kernel before
  allow_dependent_launch();

  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bars, nbox * (kWBox + hbox));
    for (int i = 0; i < nbox; ++i) {
      if (mb < 4) tma_load_2d(sbase + i * kWBox, &tmap_wd, x0 + 64 * i, 128 * mb, bars);
      else tma_load_2d(sbase + i * kWBox, &tmap_wr, x0 + 64 * i, 0, bars);
      tma_load_2d(hbase + i * hbox, &tmap_h, x0 + 64 * i, b0, bars);
    }
  }
  bool ok = true;
  if (warp < kIssuers && lane == 0) {
    const int q = warp;
    ok = wait_landed(bars, p);
    tc_fence_after();
    if (ok) {
      // K steps of 16 columns: issuer q takes [q * nbox, (q + 1) * nbox) of the 4 * nbox
      for (int kk = 0; kk < nbox; ++kk) {
        const int k = q * nbox + kk;
        const uint64_t ad = smem_desc(sbase + (k >> 2) * kWBox + (k & 3) * 32, 16, 1024, 2);
        const uint64_t bd = smem_desc(hbase + (k >> 2) * hbox + (k & 3) * 32, 16, 1024, 2);
        mma_ss(tmem + q * col_stride, ad, bd, p.idesc, kk > 0 ? 1u : 0u);
      }
      mma_commit(bars + 8 * (1 + q));
      ok = wait_landed(bars + 8 * (1 + q), p);
    } else {
      wait_landed(bars, p);   // never leave with copies in flight
    }
    ok_flags[q] = ok ? 1 : 0;
  }
  __syncthreads();
  tc_fence_after();
  ok = ok_flags[0] && ok_flags[1] && ok_flags[2] && ok_flags[3];

  // epilogue: TMEM lane = feature of the block, column = sequence; warp w reads lanes
  // [32(w%4), +32) and, of every 32 columns, the 16 of half w/4. A warp's stores for one
  // sequence cover 32 consecutive features.
  const int feat = 128 * mb + 32 * (warp & 3) + lane;
  const uint32_t lanes = (uint32_t)(32 * (warp & 3)) << 16;
  if (ok) {
    for (int c0 = 16 * (warp >> 2); c0 < p.n_tile; c0 += 32) {
      float v[16];
      uint32_t r[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) v[j] = 0.f;
      for (int q = 0; q < kIssuers; ++q) {
        tmem_ld16_sync(lanes | (tmem + q * col_stride + c0), r);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] += __uint_as_float(r[j]);
      }
      if (feat < kRow) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int b = b0 + c0 + j;
          if (c0 + j < p.n_tile && b < p.batch)
            p.part[((int64_t)kc * p.part_batch + b) * kRow + feat] = v[j];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, tmem_cols);
}

struct FinalParams {
  const float* part;
  int slices, part_batch, q_len;
  const __nv_bfloat16* gamma;
  float eps;
  const int32_t* kv_lens;
  int64_t max_kv_len;
  CacheView cv;
  __nv_bfloat16* c_kv;   // writable views of the cache rows
  __nv_bfloat16* k_r;
  uint8_t* codes;        // quantised cache (else nullptr): E4M3 codes of row r at codes + r*row_stride
  int8_t* kv_exp;        // ... and its scale exponent
  double theta[kDRope / 2];
  uint32_t* err;
};

__global__ void __launch_bounds__(kRow)
kv_finalize(const FinalParams p) {
  __shared__ float xs[kRow];
  __shared__ float red[kDLatent / 32];
  __shared__ float red_max[kRow / 32];
  // block = one (sequence, new token) row: sequence blockIdx.x / q_len, token blockIdx.x % q_len
  const int bt = blockIdx.x, b = bt / p.q_len, f = threadIdx.x, warp = f >> 5, lane = f & 31;
  grid_dependency_wait();   // the partial sums of kv_down_tc
  allow_dependent_launch();
  const int64_t L = p.kv_lens[b];
  if (L < p.q_len || L > p.max_kv_len) {   // no room for the new tokens
    if (f == 0) atomicOr(p.err, kErrBadKvLen);
    return;
  }
  const int64_t pos = L - p.q_len + bt % p.q_len;
  int64_t row;
  if (p.cv.page_table == nullptr) {
    row = (int64_t)b * p.cv.seq_stride + pos;
  } else {
    const int32_t page = p.cv.page_table[(int64_t)b * p.cv.max_pages + pos / p.cv.page_size];
    if (page < 0 || page >= p.cv.num_pages) {
      if (f == 0) atomicOr(p.err, kErrBadPage);
      return;
    }
    row = (int64_t)page * p.cv.page_size + pos % p.cv.page_size;
  }
  // the slices' partial sums, all loads in flight at once, added in slice order
  float v[kAppendSlices];
#pragma unroll
  for (int s = 0; s < kAppendSlices; ++s)
    v[s] = s < p.slices ? p.part[((int64_t)s * p.part_batch + bt) * kRow + f] : 0.f;
  float x = v[0];
#pragma unroll
  for (int s = 1; s < kAppendSlices; ++s) x += v[s];
  xs[f] = x;
  // mean square of the 512 latent features: warp sums, then the 16 warp sums in order
  float sq = f < kDLatent ? x * x : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
  if (f < kDLatent && lane == 0) red[warp] = sq;
  __syncthreads();
  double val;   // this thread's value of the row
  if (f < kDLatent) {
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kDLatent / 32; ++w) tot += red[w];
    const float y = x * rsqrtf(tot / kDLatent + p.eps) * __bfloat162float(p.gamma[f]);
    val = y;
  } else {
    // RoPE of the pair (2m, 2m+1) at the new token's position, angle reduced as in absorb
    constexpr double kTwoPiHi = 6.283185307179586;
    constexpr double kTwoPiLo = 2.4492935982947064e-16;
    constexpr double kInvTwoPi = 0.15915494309189535;
    const int i = f - kDLatent, m = i >> 1;
    const double x0 = xs[kDLatent + 2 * m], x1 = xs[kDLatent + 2 * m + 1];
    double y = (i & 1) ? x1 : x0;
    if (p.theta[m] != 0.0) {
      const double a = (double)pos * p.theta[m];
      const double k = rint(a * kInvTwoPi);
      const double r = fma(-k, kTwoPiLo, fma(-k, kTwoPiHi, a));
      double sn, cs;
      sincos(r, &sn, &cs);
      y = (i & 1) ? x0 * sn + x1 * cs : x0 * cs - x1 * sn;
    }
    val = y;
  }
  if (p.codes == nullptr) {   // bf16 row, one rounding from the computed value
    if (f < kDLatent) p.c_kv[row * p.cv.row_stride + f] = __float2bfloat16_rn((float)val);
    else p.k_r[row * p.cv.row_stride + (f - kDLatent)] = __double2bfloat16(val);
    return;
  }
  // Quantised row: the smallest power-of-two scale 2^e with max|row| / 2^e <= 448, then each
  // value / 2^e (exact) rounded to the nearest E4M3 code, ties to even.
  float am = fabsf((float)val);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  if (lane == 0) red_max[warp] = am;
  __syncthreads();
  float amax = 0.f;
#pragma unroll
  for (int w = 0; w < kRow / 32; ++w) amax = fmaxf(amax, red_max[w]);
  int e = 0;
  if (amax > 0.f) {
    e = (int)ceil(log2((double)amax / 448.0));
    while ((double)amax * exp2(-(double)e) > 448.0) ++e;
    while ((double)amax * exp2(-(double)(e - 1)) <= 448.0) --e;
    e = min(max(e, -126), 127);
  }
  const float q = (float)(val * exp2(-(double)e));
  uint32_t c2;
  asm("{ .reg .b16 t; cvt.rn.satfinite.e4m3x2.f32 t, %1, %2; cvt.u32.u16 %0, t; }" : "=r"(c2) : "f"(0.f), "f"(q));
  p.codes[row * p.cv.row_stride + f] = (uint8_t)(c2 & 0xFFu);
  if (f == 0) p.kv_exp[row] = (int8_t)e;
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// A row-major bf16 matrix [rows, cols] as a TMA source with {64 columns, box_rows} boxes,
// 128-byte swizzle (the K-major operand layout of the MMAs).
bool encode(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_append_kv(const mla_decode_s& h, int batch, int d_model,
                             const __nv_bfloat16* hidden, const __nv_bfloat16* w_dkv,
                             const __nv_bfloat16* w_kr, const __nv_bfloat16* gamma, float eps,
                             const CacheView& cv, __nv_bfloat16* c_kv, __nv_bfloat16* k_r,
                             const int32_t* kv_lens, cudaStream_t s) {
  // slices of d: at most kAppendSlices, each a multiple of 64 columns (d itself is). (Slicing
  // finer, to fill every SM, measured slower: the work is latency-bound at these sizes and
  // more slices mean more partial sums to write and add.)
  const int slice = std::max(64, (d_model / kAppendSlices + 63) / 64 * 64);
  const int rows = batch * h.q_len;   // one row per (sequence, new token)
  const int slices = (d_model + slice - 1) / slice;
  const int n_tile = std::min(64, (rows + 15) / 16 * 16);
  CUtensorMap twd, twr, th;
  if (!encode(&twd, w_dkv, kDLatent, (uint64_t)d_model, 128) ||
      !encode(&twr, w_kr, kDRope, (uint64_t)d_model, 128) ||
      !encode(&th, hidden, (uint64_t)rows, (uint64_t)d_model, (uint32_t)n_tile))
    return cudaErrorInvalidValue;
  const int nbox = slice / 64;
  const uint32_t smem = nbox * (kWBox + (uint32_t)n_tile * 128) + 128 + 1024;
  constexpr uint32_t kSmemMax = 8 * (kWBox + 64 * 128) + 128 + 1024;
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(kv_down_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemMax);
  });
  if (attr != cudaSuccess) return attr;

  DownParams dp{};
  dp.batch = rows;
  dp.n_tile = n_tile;
  dp.slice = slice;
  dp.idesc = idesc_bf16_f32(128, n_tile, false, false);
  dp.part = h.ws.append_part;
  dp.part_batch = h.cfg.max_batch * h.q_len;
  dp.err = h.ws.err;
  dp.wait_limit = 2000000000LL;
  cudaError_t e = launch_pdl(kv_down_tc, dim3(kFeatBlocks, slices, (rows + n_tile - 1) / n_tile),
                             dim3(kThreads), smem, s, twd, twr, th, dp);
  if (e != cudaSuccess) return e;

  FinalParams fp{};
  fp.part = h.ws.append_part;
  fp.slices = slices;
  fp.part_batch = h.cfg.max_batch * h.q_len;
  fp.q_len = h.q_len;
  fp.gamma = gamma;
  fp.eps = eps;
  fp.kv_lens = kv_lens;
  fp.max_kv_len = h.cfg.max_kv_len;
  fp.cv = cv;
  fp.c_kv = c_kv;
  fp.k_r = k_r;
  if (cv.kv_exp != nullptr) {   // quantised cache: c_kv is the codes' base
    fp.codes = reinterpret_cast<uint8_t*>(c_kv);
    fp.kv_exp = const_cast<int8_t*>(cv.kv_exp);
  }
  for (int m = 0; m < kDRope / 2; ++m)
    fp.theta[m] = h.theta[m];
  fp.err = h.ws.err;
  return launch_pdl(kv_finalize, dim3(rows), dim3(kRow), 0, s, fp);
}

}  // namespace mla
