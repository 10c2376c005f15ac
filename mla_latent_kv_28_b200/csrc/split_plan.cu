// The plan kernel of the attention calls: one block builds the work plan of split-KV decode
// from kv_lens (split_plan.cuh).
#include "split_plan.cuh"

namespace mla {
namespace {

__global__ void __launch_bounds__(plan::kPlanThreads)
split_plan_kernel(const int32_t* __restrict__ kv_lens, int batch, int64_t max_kv_len,
                  int units_target, int max_splits, PlanView plan, uint32_t* err) {
  __shared__ int32_t scratch[plan::kPlanScratchInts];
  grid_dependency_wait();   // kv_lens, and the plan arrays the previous call's kernels read
  allow_dependent_launch();
  plan::build_plan(kv_lens, batch, max_kv_len, units_target, max_splits, plan, err, scratch);
}

}  // namespace

cudaError_t launch_split_plan(const mla_decode_s& h, int batch, const int32_t* kv_lens,
                              cudaStream_t s) {
  return launch_pdl(split_plan_kernel, dim3(1), dim3(plan::kPlanThreads), 0, s, kv_lens, batch,
                    (int64_t)h.cfg.max_kv_len, h.units, h.cfg.max_splits, h.ws.plan, h.ws.err);
}

}  // namespace mla
