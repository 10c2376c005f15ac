// Internal declarations shared by the kernels and the C-ABI layer of libmla_decode.so.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <utility>

#include "mla_decode.h"

namespace mla {

constexpr int kDHead = 128;    // d_h
constexpr int kDLatent = 512;  // d_c
constexpr int kDRope = 64;     // d_h^R
constexpr int kRow = kDLatent + kDRope;  // one cache row: [c^KV ; k^R]
constexpr int kMaxHeads = 128;
constexpr int kMaxRows = 1 << 20;   // attention rows per sequence (heads x new tokens)
constexpr int kMaxTokenRows = 8192;  // (sequence, new token) rows per call: max_batch x new tokens
constexpr int kMaxBatch = 1024;
constexpr int kTileTokens = 64;  // tokens per KV tile: the unit of the work plan
constexpr int kAppendSlices = 16;  // the cache write's projection is split over at most 16 slices of d

// Device error word bits (see mla_check_device_errors).
constexpr uint32_t kErrBadPage = 1u << 0;
constexpr uint32_t kErrTimeout = 1u << 1;
constexpr uint32_t kErrBadKvLen = 1u << 2;

// Work plan, written on the device by the plan kernel from kv_lens, read by the decode
// and combine kernels. The cache tokens of all sequences, cut into 64-token tiles and laid
// end to end (sequence 0's tiles first), form one "tile space" of `total_tiles` tiles.
// A unit is a contiguous range of that space [unit_begin[u], unit_begin[u+1]); the decode
// kernel's CTAs (or CTA pairs) take units in turn. A unit may span several sequences; each
// (unit, sequence) overlap is a segment with its own partial-result slot. The slots of
// sequence b are seq_slot[b] .. seq_slot[b+1]-1, in token order.
struct PlanView {
  int32_t* header;      // [0] total_tiles, [1] n_units
  int32_t* seq_tile;    // [B+1]  first tile of each sequence (prefix sum of tiles)
  int32_t* seq_slot;    // [B+1]  first slot of each sequence
  int32_t* seq_len;     // [B]    kv_len as used (clamped to 0..max_kv_len)
  int32_t* seq_unit;    // [B]    the unit that holds the sequence's first tile
  int32_t* unit_begin;  // [max_units+1]
  int32_t* unit_seq;    // [max_units] first sequence that unit u touches
};

struct Workspace {
  void* base = nullptr;
  size_t bytes = 0;
  uint32_t* err = nullptr;   // device error word
  PlanView plan{};
  float* part_o = nullptr;   // [max_slots, 128 quads, n_h, 4] partial latent outputs (normalised)
  float* part_lse = nullptr; // [max_slots, n_h]     their log-sum-exp
  float* append_part = nullptr;  // [kAppendSlices, max_batch, 576] the cache write's partial sums
  int max_units = 0;
  int max_slots = 0;
};

}  // namespace mla

struct mla_decode_s {
  mla_config_t cfg;
  int device = 0;
  int num_sms = 0;
  float scale = 0.f;
  int q_len = 1;    // new tokens per sequence per call
  int n_rows = 0;   // attention rows per sequence: n_heads * q_len (token-major)
  int group_rows = 0;   // rows per decode launch (the MMA's M = 128 at most); n_rows in groups
  double theta[mla::kDRope / 2] = {};  // RoPE pair frequencies (0: no rotation), YaRN applied
  int units = 0;  // units the balanced plan cuts the tile space into
  mla::Workspace ws;
};

namespace mla {

// Programmatic dependent launch. Every kernel of the library is launched with it, so its
// launch and set-up (barriers, tensor memory, descriptor prefetch) overlap the tail of the
// kernel before it on the stream. A kernel calls grid_dependency_wait() before it reads or
// writes any global memory that earlier work on the stream may touch; that wait returns once
// every earlier grid has completed and its writes are visible. allow_dependent_launch() lets
// the next kernel start launching; it changes nothing about what that kernel may read.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void allow_dependent_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Launchers (each returns the cudaGetLastError() of its launch).
cudaError_t launch_absorb_q(const mla_decode_s& h, int batch, const __nv_bfloat16* q_c,
                            const __nv_bfloat16* q_r, const __nv_bfloat16* w_uk,
                            const int32_t* kv_lens, __nv_bfloat16* q_abs, cudaStream_t s);
// launch_absorb_q plus, in one extra CTA beside the heads, the split-KV work plan of n_seqs
// sequences (what launch_split_plan builds), for the fused decode step.
cudaError_t launch_absorb_q_with_plan(const mla_decode_s& h, int rows, int n_seqs, const __nv_bfloat16* q_c,
                                      const __nv_bfloat16* q_r, const __nv_bfloat16* w_uk,
                                      const int32_t* kv_lens, __nv_bfloat16* q_abs, cudaStream_t s);

cudaError_t launch_split_plan(const mla_decode_s& h, int batch, const int32_t* kv_lens,
                              cudaStream_t s);

struct CacheView {
  const __nv_bfloat16* c_kv;
  const __nv_bfloat16* k_r;
  int64_t row_stride;   // elements between rows
  int64_t seq_stride;   // contiguous layout: rows between sequences
  const int32_t* page_table;  // nullptr = contiguous
  int32_t max_pages;
  int32_t num_pages;
  int32_t page_size;
  // quantised cache: c_kv / k_r point at E4M3 codes (row_stride in bytes), and row r's values
  // are 2^kv_exp[r] times its codes' values
  const int8_t* kv_exp = nullptr;
  const int32_t* kv_lens = nullptr;   // prefill: read by the kernel itself (no split plan)
};

// row_base: the first of the (at most group_rows) attention rows of each sequence this launch
// takes; the partials it writes hold just those rows.
cudaError_t launch_decode_split(const mla_decode_s& h, int batch, const __nv_bfloat16* q_abs,
                                const CacheView& cache, int row_base, cudaStream_t s);

// Prefill: attention of the handle's q_len new tokens of every sequence over its cache rows,
// one work item (one head, 128 consecutive tokens) per cluster at a time; the normalised latent
// rows [B, T, n_h, 512] and lse [B, T, n_h] (or nullptr) are written directly.
cudaError_t launch_prefill(const mla_decode_s& h, int batch, const __nv_bfloat16* q_abs,
                           const CacheView& cv, __nv_bfloat16* out_latent, float* lse, cudaStream_t s);

cudaError_t launch_combine(const mla_decode_s& h, int batch, __nv_bfloat16* out_latent,
                           float* lse, int row_base, cudaStream_t s);

cudaError_t launch_combine_f32(const mla_decode_s& h, int batch, float* out_latent, float* lse,
                               int row_base, cudaStream_t s);

cudaError_t launch_merge_parts(const mla_decode_s& h, int batch, int n_parts, const float* latent_parts,
                               const float* lse_parts, __nv_bfloat16* out_latent, float* lse_out,
                               cudaStream_t s);

cudaError_t launch_append_kv(const mla_decode_s& h, int batch, int d_model,
                             const __nv_bfloat16* hidden, const __nv_bfloat16* w_dkv,
                             const __nv_bfloat16* w_kr, const __nv_bfloat16* gamma, float eps,
                             const CacheView& cv, __nv_bfloat16* c_kv, __nv_bfloat16* k_r,
                             const int32_t* kv_lens, cudaStream_t s);

cudaError_t launch_apply_wuv(const mla_decode_s& h, int batch, const __nv_bfloat16* latent,
                             const __nv_bfloat16* w_uv, __nv_bfloat16* out, cudaStream_t s);

// FP8 weights: E4M3 codes [n_h * 128, 512] and one power-of-two exponent per 1 x 128 tile
// [n_h * 128, 4] (the tile of row r covering latent columns [128 t, 128 t + 128)).
cudaError_t launch_absorb_q_fp8(const mla_decode_s& h, int batch, const __nv_bfloat16* q_c,
                                const __nv_bfloat16* q_r, const uint8_t* w_uk_codes,
                                const int8_t* w_uk_exp, const int32_t* kv_lens,
                                __nv_bfloat16* q_abs, cudaStream_t s);

cudaError_t launch_apply_wuv_fp8(const mla_decode_s& h, int batch, const __nv_bfloat16* latent,
                                 const uint8_t* w_uv_codes, const int8_t* w_uv_exp,
                                 __nv_bfloat16* out, cudaStream_t s);

}  // namespace mla
