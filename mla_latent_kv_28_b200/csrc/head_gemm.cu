// The two per-head projections of the decode step on the sm_100a tensor core:
//
//   absorb (query absorption + RoPE):  q_abs[b,i,0:512]  = W_UK,i^T q^C_{b,i}
//                                      q_abs[b,i,512:]   = RoPE_{kv_len[b]-1}(q^R_{b,i})
//   W_UV up-projection:                out[b,i,:]        = W_UV,i latent[b,i,:]
//
// Both are a small batch of vectors times one 128x512 bf16 weight matrix per head, so they
// are bound by reading the weights (16 MiB each at 128 heads). One CTA per (head, batch
// chunk) pulls its head's 128 KB of weights with TMA and runs the product as tcgen05 MMAs
// with the weights as the M = 128 operand ("swap AB": M = output features, N = batch). A
// single thread issues a small-N MMA only every ~80 cycles, so four warps issue in parallel
// into separate accumulators: one 128-feature block each for the absorption, one quarter of
// the 512-long reduction each for W_UV (the epilogue adds the four). In W_UV each issuer's
// quarter of the operands lands on a barrier of its own, so its MMAs start before the rest has
// landed. The absorption rotates q^R (brought by TMA ahead of the weights) while the weights
// land. The tile leaves tensor memory through shared memory and TMA stores, block by block.
//
// FP8 weights: E4M3 codes with one power-of-two scale 2^e per 1 x 128 tile of a weight row
// (row r of the [n_h * 128, 512] matrix, latent columns [128 t, 128 t + 128)). The codes of each
// 64-column box land by TMA in the upper half of that box's bf16 slot and all threads expand
// them in place, four boxes at a time (every thread reads its codes of the four boxes, the CTA
// meets, then the threads write the bf16 rows): E4M3 values times a power of two are exact in
// bf16, so the MMAs see exactly the dequantised weights and accumulate in fp32 as with bf16.
// The two halves land on separate barriers: the first four boxes are expanded, and the two
// issuers that need only them start their MMAs, while the other four are still landing.
#include <cudaTypedefs.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "e4m3_bf16.cuh"
#include "mla_internal.cuh"
#include "sm100.cuh"
#include "split_plan.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kThreads = 256;   // 8 warps: 4 MMA issuers, all 8 in the epilogue
constexpr int kIssuers = 4;
constexpr uint32_t kWeightBox = 128 * 128;      // 128 rows x 64 columns bf16 = 16 KB
constexpr uint32_t kWeightBytes = 8 * kWeightBox;  // one head's 128 x 512 matrix
constexpr uint32_t kCodeBox = kWeightBox / 2;      // FP8: 128 rows x 64 codes of one box

enum Mode { kAbsorb = 0, kUpProject = 1 };

struct GemmParams {
  int batch, n_heads, n_tile;     // n_tile: rows per CTA (multiple of 16, <= 128); a row is
  int q_len;                      // one (sequence, new token): row = sequence * q_len + token
  uint32_t idesc;
  __nv_bfloat16* out;             // q_abs [B, n_h, 576] or out [B, n_h, 128]
  const int8_t* w_exp;            // FP8: exponents [n_h * 128, 4]
  const __nv_bfloat16* q_r;       // absorb only
  const int32_t* kv_lens;         // absorb only
  double theta[kDRope / 2];       // absorb only: RoPE frequencies base^(-2m/d_R), 0 when off
  uint32_t* err;
  long long wait_limit;
  // fused decode step (absorb only): one extra column of CTAs, blockIdx.x == n_heads, of which
  // the first builds the split-KV work plan beside the heads
  int plan_seqs;                  // sequences; 0: no plan CTA
  int plan_units, plan_max_splits;
  int64_t plan_max_kv_len;
  PlanView plan;
};

__device__ __forceinline__ bool wait_simple(uint32_t bar, uint32_t parity, const GemmParams& p) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > p.wait_limit) {
      atomicOr(p.err, kErrTimeout);
      return false;
    }
  }
  return true;
}

constexpr int kRopeRows = 128 / (kThreads / 32);   // rows of a tile per warp (n_tile <= 128)

// The kv_len behind each of this thread's RoPE rows (rows w, w + 8, ... of the tile for warp w),
// loaded before any wait and not used until the rotation, so that the loads are in flight
// while the weights land instead of holding the thread.
__device__ __forceinline__ void rope_lens(const GemmParams& p, int b0, int (&len)[kRopeRows]) {
  const int w = threadIdx.x >> 5;
#pragma unroll
  for (int k = 0; k < kRopeRows; ++k) {
    const int r = w + 8 * k, b = b0 + r;
    len[k] = 0;
    if (r < p.n_tile && b < p.batch) len[k] = p.kv_lens[p.q_len == 1 ? b : b / p.q_len];
  }
}

// RoPE of the decoupled query of this head for the CTA's rows, from the tile of q^R that landed
// in shared memory (row r: 64 values, 128 bytes at qr + 128 r), rotated to the row's token
// position max(kv_len - q_len + token, 0) (kv_len - 1 for one new token).
// The angle pos * theta_m reaches ~1.3e5 rad at 128K tokens, so it is formed in double and
// brought into [-pi, pi] by Cody-Waite reduction with a two-term 2*pi; everything after that is
// single precision: the sine and cosine of the reduced angle (MUFU, absolute error about
// 2^-21) and the rotation by two fused multiply-adds, far below the bf16 rounding of the
// result. Lane m of warp w takes the pair (2m, 2m+1) of rows w, w + 8, ... (a warp covers one
// 128-byte row per step).
__device__ __forceinline__ void rope_rows(const GemmParams& p, int h, int b0, const uint8_t* qr,
                                          const int (&len)[kRopeRows]) {
  constexpr double kTwoPiHi = 6.283185307179586;            // nearest double to 2*pi
  constexpr double kTwoPiLo = 2.4492935982947064e-16;       // 2*pi - kTwoPiHi
  constexpr double kInvTwoPi = 0.15915494309189535;
  static_assert(kDRope / 2 == 32, "one lane per rotated pair");
  const int m = threadIdx.x & 31, w = threadIdx.x >> 5;
  const double theta = p.theta[m];
#pragma unroll
  for (int k = 0; k < kRopeRows; ++k) {
    const int r = w + 8 * k, b = b0 + r;
    if (r >= p.n_tile || b >= p.batch) break;
    const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(qr + r * 128 + 4 * m);
    float y0 = __low2float(x), y1 = __high2float(x);
    if (theta != 0.0) {
      const int pos = max(len[k] - p.q_len + (p.q_len == 1 ? 0 : b % p.q_len), 0);   // row b: token b % q_len
      const double a = (double)pos * theta;
      const double kq = rint(a * kInvTwoPi);
      const float rr = (float)fma(-kq, kTwoPiLo, fma(-kq, kTwoPiHi, a));
      float sn, cs;
      __sincosf(rr, &sn, &cs);
      const float x0 = y0, x1 = y1;
      y0 = fmaf(x0, cs, -x1 * sn);
      y1 = fmaf(x0, sn, x1 * cs);
    }
    *reinterpret_cast<__nv_bfloat162*>(p.out + ((int64_t)b * p.n_heads + h) * kRow + kDLatent + 2 * m) =
        __floats2bfloat162_rn(y0, y1);
  }
}

// FP8: bf16 boxes 4 round .. 4 round + 3 from the codes c[i] of this thread's 32 columns of box
// 4 round + i (row t / 2, half t % 2), tile scales 2^e[0] (boxes 0-1 of the round) and 2^e[1];
// kWide: an exponent above kE4m3OneMulMaxExp (two multiplies per pair, same bits).
template <bool kWide>
__device__ __forceinline__ void write_round(uint8_t* smem, const uint4 (&c)[4][2], int round, const int (&e)[2]) {
  const int t = threadIdx.x, row = t >> 1, half = t & 1;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const E4m3Scale s = e4m3_scale<kWide>(e[i >> 1]);
#pragma unroll
    for (int k = 0; k < 4; ++k) {   // 16-byte chunk half * 4 + k of the row: 8 columns
      const uint4 w = c[i][k >> 1];
      const uint32_t lo = (k & 1) ? w.z : w.x, hi = (k & 1) ? w.w : w.y;
      const int chunk = half * 4 + k;
      *reinterpret_cast<uint4*>(smem + (4 * round + i) * kWeightBox + row * 128 + ((chunk ^ (row & 7)) << 4)) =
          e4m3x8_bf16x8<kWide>(lo, hi, s);
    }
  }
}

// FP8: the codes of boxes 4 round .. 4 round + 3 (box i's 128 rows x 64 codes in the upper
// half of bf16 box i) -> those bf16 boxes (128-byte swizzle). Thread t takes row t / 2 and the
// half t % 2 of its 64 columns (32 codes) in each box. Every thread of the CTA calls it.
__device__ __forceinline__ void expand_round(uint8_t* smem, const GemmParams& p, int h, int round) {
  const int t = threadIdx.x, row = t >> 1, half = t & 1;
  uint4 c[4][2];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int k = 0; k < 2; ++k)
      c[i][k] = *reinterpret_cast<const uint4*>(smem + (4 * round + i) * kWeightBox + kCodeBox + row * 64 + half * 32 + 16 * k);
  int e[2];
#pragma unroll
  for (int q = 0; q < 2; ++q)   // the two 128-column tiles of this round's boxes
    e[q] = min(max((int)p.w_exp[((int64_t)h * kDHead + row) * (kDLatent / 128) + 2 * round + q], -126), 127);
  __syncthreads();   // every code of these boxes is read before any of them is overwritten
  if (e[0] <= kE4m3OneMulMaxExp && e[1] <= kE4m3OneMulMaxExp) write_round<false>(smem, c, round, e);
  else write_round<true>(smem, c, round, e);
  fence_proxy_async_smem();   // read by the MMAs (async proxy)
}

template <int MODE, bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
head_gemm_tc(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
             const __grid_constant__ CUtensorMap tmap_o, const __grid_constant__ CUtensorMap tmap_r,
             const GemmParams p) {
  // MODE kAbsorb:    D[c, b] = sum_d W_UK[h][d][c] x[b][d]   (A = W_UK, M-major; 4 M blocks, K = 128)
  // MODE kUpProject: D[d, b] = sum_c W_UV[h][d][c] x[b][c]   (A = W_UV, K-major; 1 M block,  K = 512)
  constexpr int kMBlocks = MODE == kAbsorb ? 4 : 1;
  constexpr int kXBoxes = MODE == kAbsorb ? 2 : 8;   // 64-column boxes of one x row
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (MODE == kAbsorb && p.plan_seqs > 0 && (int)blockIdx.x == p.n_heads) {
    // the fused step's work plan (from kv_lens), built while the heads run
    static_assert(kThreads == plan::kPlanThreads, "one block builds the plan");
    grid_dependency_wait();   // kv_lens, and the plan arrays the previous step's kernels read
    allow_dependent_launch();
    if (blockIdx.y == 0)
      plan::build_plan(p.kv_lens, p.plan_seqs, p.plan_max_kv_len, p.plan_units, p.plan_max_splits, p.plan,
                       p.err, reinterpret_cast<int32_t*>(smem));
    return;
  }
  const uint32_t sbase = smem_u32(smem);
  const uint32_t xbase = sbase + kWeightBytes;
  const uint32_t xbox = (uint32_t)p.n_tile * 128;        // bytes of one x box
  // absorb: the tile's q^R rows (n_tile x 64 bf16, unswizzled) after the x boxes
  const uint32_t qrbase = xbase + kXBoxes * xbox;
  const uint32_t bars = qrbase + (MODE == kAbsorb ? xbox : 0u);
  // barriers: [0] operands landed (FP8: x and the first four code boxes; bf16 W_UV: issuer 0's
  // weight and x boxes), [1..4] the MMAs of issuer q done, [5] FP8: the last four code boxes
  // landed, [6] absorb: q^R landed, [7..9] bf16 W_UV: issuer 1..3's weight and x boxes landed;
  // then the TMEM slot and the issuers' flags
  const uint32_t bar_hi = bars + 8 * (1 + kIssuers);
  const uint32_t bar_qr = bars + 8 * (2 + kIssuers);
  auto bar_in = [&](int q) { return q == 0 ? bars : bars + 8 * (2 + kIssuers + q); };
  // bf16 W_UV: each issuer starts once its own quarter of the operands is in (the absorption's
  // issuers rotate q^R until about when the weights have landed, so it keeps one barrier)
  constexpr bool kSplitIn = !FP8 && MODE == kUpProject;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + (bars - sbase) + 8 * (6 + kIssuers));
  const int h = blockIdx.x, b0 = blockIdx.y * p.n_tile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // accumulator block mb sits at column mb * col_stride; the epilogue reads 32 columns at a
  // time, so a block never spans fewer than 32 allocated columns
  const uint32_t col_stride = p.n_tile < 32 ? 32u : (uint32_t)p.n_tile;
  const uint32_t need = kIssuers * col_stride;   // one accumulator per issuer
  const uint32_t tmem_cols = need <= 32 ? 32 : need <= 64 ? 64 : need <= 128 ? 128 : need <= 256 ? 256 : 512;

  if (threadIdx.x == 0) {
    mbar_init(bars, 1);                                             // operands landed
    for (int q = 0; q < kIssuers; ++q) mbar_init(bars + 8 * (1 + q), 1);  // issuer q's MMAs done
    mbar_init(bar_hi, 1);
    mbar_init(bar_qr, 1);
    for (int q = 1; q < kIssuers; ++q) mbar_init(bar_in(q), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_tmap(&tmap_w);
    prefetch_tmap(&tmap_x);
    prefetch_tmap(&tmap_o);
    if (MODE == kAbsorb) prefetch_tmap(&tmap_r);
    // the head's weights into L2 while the previous kernel finishes (a hint only: L2 is
    // where writes land, so it cannot return stale data)
    for (int i = 0; i < 8; ++i) tma_prefetch_2d(&tmap_w, 64 * i, 128 * h);   // FP8: 64 codes per box
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dependency_wait();   // inputs may come from the kernel before; outputs may be read by it
  allow_dependent_launch();

  bool ok = true;
  // absorb: the rows' kv_lens are requested before the weights, so that they do not queue
  // behind this SM's 128 KB of weight copies; q^R comes first on a barrier of its own, and the
  // rotation runs while the weights are landing
  int lens[kRopeRows];
  if (MODE == kAbsorb) {
    rope_lens(p, b0, lens);
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    if (MODE == kAbsorb) {
      mbar_arrive_expect_tx(bar_qr, xbox);
      tma_load_2d(qrbase, &tmap_r, h * kDRope, b0, bar_qr);
    }
    const int xcol = h * (MODE == kAbsorb ? kDHead : kDLatent);
    if (kSplitIn) {   // quarter q: x boxes 2q, 2q+1 and weight boxes 2q, 2q+1
      for (int q = 0; q < kIssuers; ++q) {
        mbar_arrive_expect_tx(bar_in(q), 2 * kWeightBox + 2 * xbox);
        for (int i = 2 * q; i < 2 * q + 2; ++i) {
          tma_load_2d(xbase + i * xbox, &tmap_x, xcol + 64 * i, b0, bar_in(q));
          tma_load_2d(sbase + i * kWeightBox, &tmap_w, 64 * i, 128 * h, bar_in(q));
        }
      }
    } else {
      mbar_arrive_expect_tx(bars, (FP8 ? 4 * kCodeBox : kWeightBytes) + kXBoxes * xbox);
      if (FP8) mbar_arrive_expect_tx(bar_hi, 4 * kCodeBox);
      for (int i = 0; i < kXBoxes; ++i) tma_load_2d(xbase + i * xbox, &tmap_x, xcol + 64 * i, b0, bars);
      for (int i = 0; i < 8; ++i)
        tma_load_2d(sbase + i * kWeightBox + (FP8 ? kCodeBox : 0), &tmap_w, 64 * i, 128 * h,
                    FP8 && i >= 4 ? bar_hi : bars);
    }
  }
  if (MODE == kAbsorb) {
    if (wait_simple(bar_qr, 0, p)) rope_rows(p, h, b0, smem + (qrbase - sbase), lens);
    else if (threadIdx.x == 0) wait_simple(bar_qr, 0, p);   // never leave with the copy in flight
  }
  volatile int* ok_flags = reinterpret_cast<volatile int*>(smem + (bars - sbase) + 8 * (6 + kIssuers) + 4);
  // issuer q's MMAs: absorb: accumulator q = output features [128q, 128q+128), K = 128 (8
  // steps); W_UV: accumulator q = the partial sum over latent columns [128q, 128q+128). Either
  // way they read weight boxes 2q and 2q+1 only.
  auto issue = [&](int q) {
    tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        uint64_t ad, bd;
        if (MODE == kAbsorb) {
          // A[c, d]: W_UK box (2q) holds d rows x 64 c; 16 d rows per K step
          ad = smem_desc(sbase + 2 * q * kWeightBox + kk * 2048, kWeightBox, 1024, 2);
          bd = smem_desc(xbase + (kk >> 2) * xbox + (kk & 3) * 32, 16, 1024, 2);
        } else {
          const int k = 8 * q + kk;   // K step over the 512 latent columns
          ad = smem_desc(sbase + (k >> 2) * kWeightBox + (k & 3) * 32, 16, 1024, 2);
          bd = smem_desc(xbase + (k >> 2) * xbox + (k & 3) * 32, 16, 1024, 2);
        }
        mma_ss(tmem + q * col_stride, ad, bd, p.idesc, kk > 0 ? 1u : 0u);
    }
    mma_commit(bars + 8 * (1 + q));
  };
  bool issued = false;   // issuer threads: this thread's MMAs are in flight
  if (FP8) {
    // every thread expands its share of boxes 0..3 once they land, then issuers 0 and 1 (which
    // read only those) start while boxes 4..7 are expanded, then issuers 2 and 3
    bool good = true;
    for (int round = 0; round < 2; ++round) {
      const bool landed = wait_simple(round == 0 ? bars : bar_hi, 0, p);
      good = __syncthreads_and(good && landed ? 1 : 0) != 0;
      if (!good) continue;
      expand_round(smem, p, h, round);
      __syncthreads();
      if (warp < kIssuers && lane == 0 && (warp >> 1) == round) {
        issue(warp);
        issued = true;
      }
    }
    if (!good && threadIdx.x == 0) {   // never leave with copies in flight
      wait_simple(bars, 0, p);
      wait_simple(bar_hi, 0, p);
    }
  }
  if (!FP8 && warp < kIssuers && lane == 0) {
    const uint32_t in = kSplitIn ? bar_in(warp) : bars;
    issued = wait_simple(in, 0, p);
    if (issued) issue(warp);
    else wait_simple(in, 0, p);   // never leave with copies in flight
  }
  if (warp < kIssuers && lane == 0) {
    ok = issued && wait_simple(bars + 8 * (1 + warp), 0, p);
    ok_flags[warp] = ok ? 1 : 0;
  }
  __syncthreads();
  tc_fence_after();
  ok = ok_flags[0] && ok_flags[1] && ok_flags[2] && ok_flags[3];

  // epilogue: TMEM lane = output feature, column = sequence. The tile goes out through
  // shared memory (the weights' buffer, free once the MMAs are done) as boxes of 64 features
  // x n_tile sequences, written by TMA: a warp's direct stores would each cover only the
  // 64 bytes of one output row.
  // Warp w reads TMEM lanes [32(w%4), +32) and, of every 32 columns, the 16 of half w/4.
  const uint32_t lanes = (uint32_t)(32 * (warp & 3)) << 16;
  const int chalf = 16 * (warp >> 2);
  const uint32_t obox = (uint32_t)p.n_tile * 128;   // bytes of one 64-feature output box
  // (ok is the same for the whole CTA.) Each block of 128 features is stored as soon as it is
  // written, so its TMA stores overlap the next block's reads of tensor memory.
  const int x0 = h * (MODE == kAbsorb ? kRow : kDHead);
  for (int mb = 0; mb < kMBlocks && ok; ++mb) {
    const int feat = 128 * mb + 32 * (warp & 3) + lane;
    uint8_t* col = smem + (feat >> 6) * obox + (feat & 63) * 2;
    for (int c0 = chalf; c0 < p.n_tile; c0 += 32) {
      float v[16];
      uint32_t r[16];
      if (MODE == kAbsorb) {
        tmem_ld16_sync(lanes | (tmem + mb * col_stride + c0), r);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0.f;
        for (int q = 0; q < kIssuers; ++q) {   // the four partial sums over the latent columns
          tmem_ld16_sync(lanes | (tmem + q * col_stride + c0), r);
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] += __uint_as_float(r[j]);
        }
      }
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (c0 + j < p.n_tile)
          *reinterpret_cast<__nv_bfloat16*>(col + (c0 + j) * 128) = __float2bfloat16_rn(v[j]);
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int k = 2 * mb; k < 2 * mb + 2; ++k) tma_store_2d(&tmap_o, sbase + k * obox, x0 + 64 * k, b0);
      bulk_commit_group();
    }
  }
  if (ok && threadIdx.x == 0) bulk_wait_group0();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, tmem_cols);
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

// A row-major bf16 matrix [rows, cols] as a TMA source or destination with 64-column boxes.
bool encode(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
            CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The FP8 weight codes [rows, 512] bytes as a TMA source with {64, 128} boxes (no swizzle).
bool encode_codes(CUtensorMap* m, const void* base, uint64_t rows) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kDLatent, rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kDLatent};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// plan_seqs > 0 (absorb only): also build the split-KV work plan for that many sequences, in one
// extra CTA.
template <int MODE, bool FP8>
cudaError_t launch(const mla_decode_s& h, int batch, const void* w, const int8_t* w_exp,
                   const __nv_bfloat16* x, __nv_bfloat16* out, const __nv_bfloat16* q_r,
                   const int32_t* kv_lens, cudaStream_t s, int plan_seqs = 0) {
  constexpr int kXBoxes = MODE == kAbsorb ? 2 : 8;
  constexpr int kCap = MODE == kAbsorb ? 128 : 64;  // weights + x boxes fit in shared memory
  const int n_tile = std::min(kCap, (batch + 15) / 16 * 16);
  const int kx = MODE == kAbsorb ? kDHead : kDLatent;
  const int ko = MODE == kAbsorb ? kRow : kDHead;   // output row of one head
  CUtensorMap tw, tx, to, tr;
  const bool w_ok = FP8 ? encode_codes(&tw, w, (uint64_t)h.cfg.n_heads * kDHead)
                        : encode(&tw, w, (uint64_t)h.cfg.n_heads * kDHead, kDLatent, 128);
  if (!w_ok ||
      !encode(&tx, x, (uint64_t)batch, (uint64_t)h.cfg.n_heads * kx, (uint32_t)n_tile) ||
      !encode(&to, out, (uint64_t)batch, (uint64_t)h.cfg.n_heads * ko, (uint32_t)n_tile,
              CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  // absorb: q^R [rows, n_h * 64] in boxes of 64 values x n_tile rows (W_UV: unused)
  tr = tx;
  if (MODE == kAbsorb && !encode(&tr, q_r, (uint64_t)batch, (uint64_t)h.cfg.n_heads * kDRope,
                                 (uint32_t)n_tile, CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  constexpr int kBoxes = kXBoxes + (MODE == kAbsorb ? 1 : 0);   // x boxes, and absorb's q^R box
  constexpr uint32_t kSmemMax = kWeightBytes + kBoxes * kCap * 128 + 128 + 1024;
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(head_gemm_tc<MODE, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kSmemMax);
  });
  if (attr != cudaSuccess) return attr;
  GemmParams p{};
  p.batch = batch;
  p.n_heads = h.cfg.n_heads;
  p.n_tile = n_tile;
  p.q_len = h.q_len;
  p.idesc = idesc_bf16_f32(128, n_tile, MODE == kAbsorb, false);
  p.out = out;
  p.w_exp = w_exp;
  p.q_r = q_r;
  p.kv_lens = kv_lens;
  for (int m = 0; m < kDRope / 2; ++m)
    p.theta[m] = h.theta[m];
  p.err = h.ws.err;
  p.wait_limit = 2000000000LL;
  p.plan_seqs = MODE == kAbsorb ? plan_seqs : 0;
  p.plan_units = h.units;
  p.plan_max_splits = h.cfg.max_splits;
  p.plan_max_kv_len = h.cfg.max_kv_len;
  p.plan = h.ws.plan;
  const uint32_t smem = kWeightBytes + kBoxes * n_tile * 128 + 128 + 1024;
  static_assert(kWeightBytes >= plan::kPlanScratchInts * 4, "the plan CTA's scratch fits");
  dim3 grid(h.cfg.n_heads + (p.plan_seqs > 0 ? 1 : 0), (batch + n_tile - 1) / n_tile);
  return launch_pdl(head_gemm_tc<MODE, FP8>, grid, dim3(kThreads), smem, s, tw, tx, to, tr, p);
}

}  // namespace

cudaError_t launch_absorb_q(const mla_decode_s& h, int batch, const __nv_bfloat16* q_c,
                            const __nv_bfloat16* q_r, const __nv_bfloat16* w_uk,
                            const int32_t* kv_lens, __nv_bfloat16* q_abs, cudaStream_t s) {
  return launch<kAbsorb, false>(h, batch, w_uk, nullptr, q_c, q_abs, q_r, kv_lens, s);
}

cudaError_t launch_absorb_q_with_plan(const mla_decode_s& h, int rows, int n_seqs, const __nv_bfloat16* q_c,
                                      const __nv_bfloat16* q_r, const __nv_bfloat16* w_uk,
                                      const int32_t* kv_lens, __nv_bfloat16* q_abs, cudaStream_t s) {
  return launch<kAbsorb, false>(h, rows, w_uk, nullptr, q_c, q_abs, q_r, kv_lens, s, n_seqs);
}

cudaError_t launch_apply_wuv(const mla_decode_s& h, int batch, const __nv_bfloat16* latent,
                             const __nv_bfloat16* w_uv, __nv_bfloat16* out, cudaStream_t s) {
  return launch<kUpProject, false>(h, batch, w_uv, nullptr, latent, out, nullptr, nullptr, s);
}

cudaError_t launch_absorb_q_fp8(const mla_decode_s& h, int batch, const __nv_bfloat16* q_c,
                                const __nv_bfloat16* q_r, const uint8_t* w_uk_codes,
                                const int8_t* w_uk_exp, const int32_t* kv_lens,
                                __nv_bfloat16* q_abs, cudaStream_t s) {
  return launch<kAbsorb, true>(h, batch, w_uk_codes, w_uk_exp, q_c, q_abs, q_r, kv_lens, s);
}

cudaError_t launch_apply_wuv_fp8(const mla_decode_s& h, int batch, const __nv_bfloat16* latent,
                                 const uint8_t* w_uv_codes, const int8_t* w_uv_exp,
                                 __nv_bfloat16* out, cudaStream_t s) {
  return launch<kUpProject, true>(h, batch, w_uv_codes, w_uv_exp, latent, out, nullptr, nullptr, s);
}

}  // namespace mla
