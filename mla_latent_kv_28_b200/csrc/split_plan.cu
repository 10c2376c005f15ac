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
#include "mla_internal.cuh"

namespace mla {
namespace {

__device__ int upper_index(const int32_t* v, int n, int t) {
  // largest i in [0, n) with v[i] <= t (v non-decreasing, v[0] <= t)
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (v[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(256)
split_plan_kernel(const int32_t* __restrict__ kv_lens, int batch, int64_t max_kv_len,
                  int units_target, int max_splits, PlanView plan, uint32_t* err) {
  __shared__ int32_t s_tiles[kMaxBatch];
  __shared__ int32_t s_tstart[kMaxBatch + 1];
  __shared__ int32_t s_units;
  const int tid = threadIdx.x;
  grid_dependency_wait();   // kv_lens, and the plan arrays the previous call's kernels read
  allow_dependent_launch();

  for (int b = tid; b < batch; b += blockDim.x) {
    int64_t L = kv_lens[b];
    if (L < 0 || L > max_kv_len) {
      atomicOr(err, kErrBadKvLen);
      L = L < 0 ? 0 : max_kv_len;
    }
    plan.seq_len[b] = (int32_t)L;
    s_tiles[b] = (int32_t)((L + kTileTokens - 1) / kTileTokens);
  }
  __syncthreads();

  if (tid == 0) {
    int acc = 0;
    for (int b = 0; b < batch; ++b) { s_tstart[b] = acc; acc += s_tiles[b]; }
    s_tstart[batch] = acc;
    const int total = acc;
    int n_units = 0;
    if (total > 0) {
      if (max_splits == 0) {
        const int per = (total + units_target - 1) / units_target;
        n_units = (total + per - 1) / per;
        for (int u = 0; u < n_units; ++u) plan.unit_begin[u] = u * per;
      } else {
        for (int b = 0; b < batch; ++b) {
          const int t = s_tiles[b];
          const int n = t < max_splits ? t : max_splits;
          for (int k = 0; k < n; ++k) plan.unit_begin[n_units++] = s_tstart[b] + (k * t) / n;
        }
      }
    }
    plan.unit_begin[n_units] = total;
    plan.header[0] = total;
    plan.header[1] = n_units;
    s_units = n_units;
    for (int b = 0; b <= batch; ++b) plan.seq_tile[b] = s_tstart[b];
  }
  __syncthreads();
  const int n_units = s_units;
  const int total = s_tstart[batch];

  // first sequence of each unit: the one whose tile range holds the unit's first tile
  for (int u = tid; u < n_units; u += blockDim.x)
    plan.unit_seq[u] = upper_index(s_tstart, batch, plan.unit_begin[u]);
  // first unit of each sequence, and how many units (slots) it spans
  for (int b = tid; b < batch; b += blockDim.x) {
    int n = 0, first = 0;
    if (s_tiles[b] > 0) {
      first = upper_index(plan.unit_begin, n_units, s_tstart[b]);
      const int last = upper_index(plan.unit_begin, n_units, s_tstart[b] + s_tiles[b] - 1);
      n = last - first + 1;
    }
    plan.seq_unit[b] = first;
    s_tiles[b] = n;  // reuse: slots of sequence b
  }
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int b = 0; b < batch; ++b) { plan.seq_slot[b] = acc; acc += s_tiles[b]; }
    plan.seq_slot[batch] = acc;
  }
  (void)total;
}

}  // namespace

cudaError_t launch_split_plan(const mla_decode_s& h, int batch, const int32_t* kv_lens,
                              cudaStream_t s) {
  return launch_pdl(split_plan_kernel, dim3(1), dim3(256), 0, s, kv_lens, batch,
                    (int64_t)h.cfg.max_kv_len, h.units, h.cfg.max_splits, h.ws.plan, h.ws.err);
}

}  // namespace mla
