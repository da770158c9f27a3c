// The two-term tf32 split of fp32 operands (the fp32 expert path).
//
// tf32 keeps fp32's 8-bit exponent and the top 10 bits of its mantissa.  An
// fp32 value v becomes v_hi = v rounded to tf32 (nearest, ties to even) and
// v_lo = v - v_hi.  v_lo is exact in fp32 (it is made of v's low 13 mantissa
// bits) and |v_lo| <= 2^-11 |v|, so v_hi + tf32(v_lo) equals v within
// 2^-21 |v|.  For a product w . x the expert GEMMs then accumulate the three
// terms w_hi x_hi + w_lo x_hi + w_hi x_lo (the fourth, w_lo x_lo, is below
// 2^-22 |w x|) on the tf32 tensor cores.
#pragma once

#include <cstdint>

namespace moe {

// v rounded to the nearest tf32 value (ties to even), as an fp32 whose low 13
// mantissa bits are zero.  Infinities and NaNs pass unchanged; a finite value
// that rounds past the largest finite one becomes infinity, as rounding does.
__device__ __forceinline__ float tf32_round(float v) {
  uint32_t u = __float_as_uint(v);
  if ((u & 0x7F800000u) == 0x7F800000u) return v;
  u += 0xFFFu + ((u >> 13) & 1u);
  return __uint_as_float(u & 0xFFFFE000u);
}

// (hi, lo) with hi = tf32_round(v), lo = v - hi (exact).
__device__ __forceinline__ void tf32_split(float v, float& hi, float& lo) {
  hi = tf32_round(v);
  lo = v - hi;
}

}  // namespace moe
