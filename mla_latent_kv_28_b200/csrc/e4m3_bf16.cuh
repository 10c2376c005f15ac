// E4M3 codes (OCP FP8 E4M3: sign, 4 exponent bits with bias 7, 3 mantissa bits) to bf16 values
// times a power of two 2^E, the expansion the quantised cache and the FP8 weights both use.
//
// The code's bits placed into a bf16, (s << 15) | ((c & 0x7F) << 4), are the bf16 with exponent
// field eeee and mantissa mmm0000, whose value is 2^-120 times the code's for every code: a
// normal code is 2^(e-7)(1 + m/8) against 2^(e-127)(1 + m/8), a subnormal code (e = 0) m 2^-9
// against the bf16 subnormal m 2^-129, and zero stays zero. Exact bf16 multiplies (round to
// nearest, subnormals kept) then give the nearest bf16 to 2^E times the code, which is the
// code's value exactly unless it falls below bf16's normal range: one multiply by 2^(120 + E)
// when that is a bf16 (E <= 7, every realistic row), else 2^120 and then 2^E. A pair of codes
// costs a byte permute, a shift, two logic operations and one or two bf16x2 multiplies, and no
// conversion instruction: the conversion pipe is the one the attention's exponentials and its
// float/integer conversions run on.
#pragma once

#include <cstdint>

namespace mla {

// Largest exponent E that takes a single multiply.
constexpr int kE4m3OneMulMaxExp = 7;

// bf16x2 holding 2^k in both halves, -126 <= k <= 127.
__device__ __forceinline__ uint32_t bf16x2_pow2(int k) {
  const uint32_t f = (uint32_t)(k + 127);
  return (f << 7) | (f << 23);
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// The two scale operands of a row or tile with exponent e (clamped to -126..127 by the caller).
struct E4m3Scale {
  uint32_t a, b;   // multiply by a, then (kWide) by b
};
template <bool kWide>
__device__ __forceinline__ E4m3Scale e4m3_scale(int e) {
  return kWide ? E4m3Scale{bf16x2_pow2(120), bf16x2_pow2(e)} : E4m3Scale{bf16x2_pow2(120 + e), 0u};
}

// x = (c0 << 8) | (c1 << 24) -> bf16x2 (low half c0) of the two codes times 2^E.
template <bool kWide>
__device__ __forceinline__ uint32_t e4m3x2_bf16x2(uint32_t x, E4m3Scale s) {
  const uint32_t r = ((x >> 4) & 0x07F007F0u) | (x & 0x80008000u);
  const uint32_t d = bf16x2_mul(r, s.a);
  return kWide ? bf16x2_mul(d, s.b) : d;
}

// Eight codes (lo4: codes 0-3, hi4: codes 4-7, low byte first) -> eight bf16.
template <bool kWide>
__device__ __forceinline__ uint4 e4m3x8_bf16x8(uint32_t lo4, uint32_t hi4, E4m3Scale s) {
  return make_uint4(e4m3x2_bf16x2<kWide>(__byte_perm(lo4, 0u, 0x1404u), s),
                    e4m3x2_bf16x2<kWide>(__byte_perm(lo4, 0u, 0x3424u), s),
                    e4m3x2_bf16x2<kWide>(__byte_perm(hi4, 0u, 0x1404u), s),
                    e4m3x2_bf16x2<kWide>(__byte_perm(hi4, 0u, 0x3424u), s));
}

}  // namespace mla
