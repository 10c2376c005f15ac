// In-place expansion of a quantised cache tile (E4M3 codes, one power-of-two scale per row)
// to the bf16 layout the decode kernel's MMAs read. Included by decode_split.cu inside its
// namespace, after kBoxC / kBoxR and e4m3_bf16.cuh are known.
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

// The row's codes -> bf16 (2^e times each code); kWide: e above kE4m3OneMulMaxExp (two
// multiplies per pair instead of one, same bits).
template <bool kWide>
__device__ __forceinline__ void write_row(uint8_t* stage, int t, const TileCodes& v, int e) {
  const int row = t >> 1, half = t & 1;
  const E4m3Scale s = e4m3_scale<kWide>(e);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int k = 0; k < 4; ++k) {   // 16-byte chunk half*4 + k of the row: 8 columns
      const uint4 w = v.c[i][k >> 1];
      const int chunk = half * 4 + k;
      *reinterpret_cast<uint4*>(stage + i * kBoxC + row * 128 + ((chunk ^ (row & 7)) << 4)) =
          (k & 1) ? e4m3x8_bf16x8<kWide>(w.z, w.w, s) : e4m3x8_bf16x8<kWide>(w.x, w.y, s);
    }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int chunk = half * 2 + k;
    *reinterpret_cast<uint4*>(stage + 4 * kBoxC + row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4)) =
        k ? e4m3x8_bf16x8<kWide>(v.r.z, v.r.w, s) : e4m3x8_bf16x8<kWide>(v.r.x, v.r.y, s);
  }
}

__device__ __forceinline__ void write_bf16(uint8_t* stage, int t, const TileCodes& v, int e) {
  if (e <= kE4m3OneMulMaxExp) write_row<false>(stage, t, v, e);
  else write_row<true>(stage, t, v, e);
}
