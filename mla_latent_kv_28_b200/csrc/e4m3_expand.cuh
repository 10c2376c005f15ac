// In-place expansion of a quantised cache tile (E4M3 codes, one power-of-two scale per row)
// to the bf16 layout the decode kernel's MMAs read. Included by decode_split.cu inside its
// namespace, after kBoxC / kBoxR (and cuda_fp16.h) are known.
//
// Each 64-column box's codes (64 rows x 64 bytes, landed by TMA) sit in the upper half of that
// box's bf16 slot, the k^R codes (64 rows x 32 bytes) in the upper half of the k^R slot. The
// expanding warpgroup writes them back in the layout the bf16 cache lands in (128- and
// 64-byte swizzles): every thread first reads its codes (thread t: row t/2, half t%2 of each
// box), the warpgroup meets, then the threads write, so no code is overwritten before it is
// read.
#pragma once

constexpr uint32_t kQ8StageBytes = 4 * (kBoxC / 2) + kBoxR / 2;   // 18 KB of codes per tile

struct TileCodes {
  uint4 c[4][2];   // 32 c^KV codes of each box
  uint4 r;         // 16 k^R codes
};

__device__ __forceinline__ void read_codes(const uint8_t* stage, int t, TileCodes& v) {
  const int row = t >> 1, half = t & 1;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int k = 0; k < 2; ++k)
      v.c[i][k] = *reinterpret_cast<const uint4*>(stage + i * kBoxC + kBoxC / 2 + row * 64 + half * 32 + 16 * k);
  v.r = *reinterpret_cast<const uint4*>(stage + 4 * kBoxC + kBoxR / 2 + row * 32 + half * 16);
}

// Two E4M3 codes (low byte first) -> their values times 2^e as a bf16 pair: E4M3 -> f16 by the
// hardware conversion (exact), f16 -> f32 (exact), times the power-of-two scale (exact), and
// bf16 of that (exact: 4 significant bits). (A version with shifts, logic and two multiplies
// per value instead of conversions measured slower: more instructions per value on a
// latency-bound warpgroup.)
__device__ __forceinline__ uint32_t e4m3x2_bf16x2(uint32_t codes2, float scale) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((unsigned short)(codes2 & 0xFFFFu)));
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
  __nv_bfloat162 b = __floats2bfloat162_rn(f.x * scale, f.y * scale);
  return *reinterpret_cast<uint32_t*>(&b);
}

__device__ __forceinline__ uint4 expand8(uint32_t lo4, uint32_t hi4, float scale) {
  return make_uint4(e4m3x2_bf16x2(lo4, scale), e4m3x2_bf16x2(lo4 >> 16, scale),
                    e4m3x2_bf16x2(hi4, scale), e4m3x2_bf16x2(hi4 >> 16, scale));
}

__device__ __forceinline__ void write_bf16(uint8_t* stage, int t, const TileCodes& v, float scale) {
  const int row = t >> 1, half = t & 1;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int k = 0; k < 4; ++k) {   // 16-byte chunk half*4 + k of the row: 8 columns
      const uint4 w = v.c[i][k >> 1];
      const int chunk = half * 4 + k;
      *reinterpret_cast<uint4*>(stage + i * kBoxC + row * 128 + ((chunk ^ (row & 7)) << 4)) =
          (k & 1) ? expand8(w.z, w.w, scale) : expand8(w.x, w.y, scale);
    }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int chunk = half * 2 + k;
    *reinterpret_cast<uint4*>(stage + 4 * kBoxC + row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4)) =
        k ? expand8(v.r.z, v.r.w, scale) : expand8(v.r.x, v.r.y, scale);
  }
}

