// FP8 E4M3FN weight codes -> bf16, for the weight-only FP8 expert GEMMs.
//
// An E4M3FN code is sign (bit 7), exponent e (bits 6..3, bias 7), mantissa m
// (bits 2..0): (1 + m/8) * 2^(e-7) for e >= 1, m * 2^-9 for e = 0; S.1111.111
// is NaN and there are no infinities (largest finite magnitude 448).  Every
// finite code is exactly a bf16 value (at most 4 significant bits, exponents
// -9..8).
//
// Decoding without a conversion instruction: place the code's 7 magnitude
// bits at bits 10..4 of a 16-bit half and its sign at bit 15.  Read as bf16,
// that half has exponent field e and the top three mantissa bits m, i.e. it is
// the code's value times 2^-120 (for e = 0 it is the bf16 subnormal
// m * 2^-129, again 2^-120 times m * 2^-9).  One bf16x2 multiply by 2^120 is
// exact and gives the value.  A NaN code would decode to +-480: the weight
// format excludes NaN codes.
#pragma once

#include <stdint.h>

namespace moe {

// prmt.b32 with the default mode: per destination byte, selector nibble bits
// 2..0 pick a source byte of {b, a} and bit 3 replicates that byte's sign bit.
__device__ __forceinline__ uint32_t prmt_b32(uint32_t a, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(0u), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

constexpr uint32_t kBf16x2Pow2_120 = 0x7B807B80u;  // {2^120, 2^120}
constexpr uint32_t kE4m3PlaceMask = 0x87F087F0u;   // sign bit 15, magnitude bits 10..4

// Four codes (w's bytes, lowest byte first) -> bf16x2 words lo = {code0,
// code1} and hi = {code2, code3}, low half first.
__device__ __forceinline__ void e4m3x4_to_bf16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  // bytes {c0, sign(c0), c1, sign(c1)} and {c2, sign(c2), c3, sign(c3)}
  const uint32_t a = prmt_b32(w, 0x9180u);
  const uint32_t b = prmt_b32(w, 0xB3A2u);
  lo = bf16x2_mul((a << 4) & kE4m3PlaceMask, kBf16x2Pow2_120);
  hi = bf16x2_mul((b << 4) & kE4m3PlaceMask, kBf16x2Pow2_120);
}

}  // namespace moe
