// Work plan for split-KV decode, built on the device from kv_lens (no host round trip, so
// a whole decode step can be enqueued, or captured, without a synchronisation).
//
// The cached tokens of all sequences, cut into 64-token tiles and laid end to end, form a
// tile space. Two ways to cut it into units (one unit = one CTA pair's share of work):
//   balanced (max_splits == 0): `units` equal ranges; a range may cross sequences, so a
//            ragged batch loads every pair alike whatever the length mix;
//   capped   (max_splits  > 0): every sequence alone is cut into min(max_splits, tiles)
//            near-equal ranges; a unit never crosses a sequence.
// Every (unit, sequence) overlap is a segment with its own partial slot; the slots of one
// sequence are consecutive, in token order, and the combine kernel merges them.
//
// build_plan is the plan's body: the plan kernel of the attention calls runs it, and so does one
// extra CTA of the absorption kernel in the fused decode step.
#pragma once

#include "mla_internal.cuh"

namespace mla {
namespace plan {

__device__ inline int upper_index(const int32_t* v, int n, int t) {
  // largest i in [0, n) with v[i] <= t (v non-decreasing, v[0] <= t)
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (v[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

constexpr int kPlanThreads = 256;
constexpr int kPerThread = kMaxBatch / kPlanThreads;   // sequences per thread (4)
constexpr int kPlanScratchInts = 3 * (kMaxBatch + 1) + kPlanThreads / 32 + 1;

// Exclusive prefix sum over the block of x[0..n) (n <= kMaxBatch) into out[0..n], out[n] = total.
// Each thread scans its kPerThread consecutive entries, the warps scan their threads with
// shuffles, and one warp scans the warp totals.
__device__ inline void block_exclusive_scan(const int32_t* x, int n, int32_t* out, int32_t* warp_tot) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int v[kPerThread];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) {
    const int idx = tid * kPerThread + i;
    v[i] = idx < n ? x[idx] : 0;
    sum += v[i];
  }
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int t = lane < kPlanThreads / 32 ? warp_tot[lane] : 0;
    int ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += y;
    }
    if (lane < kPlanThreads / 32) warp_tot[lane] = ti - t;   // exclusive warp offsets
    if (lane == kPlanThreads / 32 - 1) warp_tot[kPlanThreads / 32] = ti;   // total
  }
  __syncthreads();
  int run = warp_tot[warp] + incl - sum;
#pragma unroll
  for (int i = 0; i < kPerThread; ++i) {
    const int idx = tid * kPerThread + i;
    if (idx < n) out[idx] = run;
    run += v[i];
  }
  if (tid == 0) out[n] = warp_tot[kPlanThreads / 32];
  __syncthreads();
}

// The plan from kv_lens, by one block of kPlanThreads threads, with kPlanScratchInts ints of
// this block's shared memory as scratch. The caller has waited for the kernels that write
// kv_lens or read the plan arrays.
__device__ inline void build_plan(const int32_t* __restrict__ kv_lens, int batch, int64_t max_kv_len,
                                  int units_target, int max_splits, PlanView plan, uint32_t* err,
                                  int32_t* scratch) {
  int32_t* s_a = scratch;                           // [kMaxBatch + 1] per-sequence counts
  int32_t* s_tstart = s_a + (kMaxBatch + 1);         // [kMaxBatch + 1]
  int32_t* s_aux = s_tstart + (kMaxBatch + 1);       // [kMaxBatch + 1]
  int32_t* s_warp = s_aux + (kMaxBatch + 1);         // [kPlanThreads / 32 + 1]
  const int tid = threadIdx.x;

  for (int b = tid; b < batch; b += kPlanThreads) {
    int64_t L = kv_lens[b];
    if (L < 0 || L > max_kv_len) {
      atomicOr(err, kErrBadKvLen);
      L = L < 0 ? 0 : max_kv_len;
    }
    plan.seq_len[b] = (int32_t)L;
    s_a[b] = (int32_t)((L + kTileTokens - 1) / kTileTokens);   // tiles of sequence b
  }
  __syncthreads();
  block_exclusive_scan(s_a, batch, s_tstart, s_warp);
  const int total = s_tstart[batch];
  for (int b = tid; b <= batch; b += kPlanThreads) plan.seq_tile[b] = s_tstart[b];

  int n_units = 0, per = 0;
  if (total > 0) {
    if (max_splits == 0) {
      per = (total + units_target - 1) / units_target;
      n_units = (total + per - 1) / per;
      for (int u = tid; u < n_units; u += kPlanThreads) {
        plan.unit_begin[u] = u * per;
        // first sequence of the unit: the one whose tile range holds its first tile
        plan.unit_seq[u] = upper_index(s_tstart, batch, u * per);
      }
    } else {
      // sequence b is cut into min(max_splits, tiles) near-equal ranges, units s_aux[b] on
      for (int b = tid; b < batch; b += kPlanThreads) s_aux[b] = min(s_a[b], max_splits);
      __syncthreads();
      block_exclusive_scan(s_aux, batch, s_aux, s_warp);
      n_units = s_aux[batch];
      for (int b = tid; b < batch; b += kPlanThreads) {
        const int t = s_a[b], n = min(t, max_splits);
        for (int k = 0; k < n; ++k) {
          plan.unit_begin[s_aux[b] + k] = s_tstart[b] + (k * t) / n;
          plan.unit_seq[s_aux[b] + k] = b;
        }
      }
    }
  }
  if (tid == 0) {
    plan.unit_begin[n_units] = total;
    plan.header[0] = total;
    plan.header[1] = n_units;
  }

  // first unit of each sequence and how many units (slots) it spans, from the cut itself
  // (no search of unit_begin in global memory): balanced units are per tiles long; capped
  // units never cross a sequence
  for (int b = tid; b < batch; b += kPlanThreads) {
    int n = 0, first = 0;
    if (s_a[b] > 0) {
      if (max_splits == 0) {
        first = s_tstart[b] / per;
        n = (s_tstart[b] + s_a[b] - 1) / per - first + 1;
      } else {
        first = s_aux[b];
        n = min(s_a[b], max_splits);
      }
    }
    plan.seq_unit[b] = first;
    s_aux[b] = n;   // slots of sequence b
  }
  __syncthreads();
  block_exclusive_scan(s_aux, batch, s_aux, s_warp);
  for (int b = tid; b <= batch; b += kPlanThreads) plan.seq_slot[b] = s_aux[b];
}


}  // namespace plan
}  // namespace mla
