// Device pieces of the CTA-pair (2-SM UMMA) GEMM mainloop shared by the
// standalone pair GEMMs (grouped_gemm_pair.cu) and the fused persistent MoE
// kernel (fused_moe.cu): the stage layout, the narrow-tile rule and the
// unrolled MMA issue of one stage.
#pragma once

#include "gemm_common.cuh"
#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {
namespace gemm {

constexpr int kPairBN = 256;  // tokens per tile (the pair MMA's N)

// One pipeline slot of a CTA of the pair: K sub-blocks of 64 (one 128-byte
// swizzled row each) of this CTA's 128 weight rows (A) and of its token half
// (B).  A wide stage holds 2 sub-blocks of A and 2 of 128 token rows; a
// narrow stage (token half <= 32 rows) 3 sub-blocks of A and 3 of 32 rows.
struct PairStage {
  static constexpr int ROW = kBK * 2;                    // bytes per 64-element swizzled row
  static constexpr int SUB_A = kBM * ROW;                // one 64-K sub-block of this CTA's A
  static constexpr int SUB_BW = (kPairBN / 2) * ROW;     // ... of this CTA's B, wide tile
  static constexpr int SUB_BN = kBBoxRows * ROW;         // ... of this CTA's B, narrow tile
  static constexpr int KS_W = 2;                         // K sub-blocks per wide stage
  static constexpr int KS_N = 3;                         // K sub-blocks per narrow stage
  static constexpr int B_OFF_W = KS_W * SUB_A;           // B within a wide stage
  static constexpr int B_OFF_N = KS_N * SUB_A;           // B within a narrow stage
  static constexpr int A_BYTES_W = KS_W * SUB_A;         // one CTA's A bytes per stage
  static constexpr int A_BYTES_N = KS_N * SUB_A;
  static constexpr int B_BYTES_W = KS_W * SUB_BW;        // one CTA's B bytes per stage
  static constexpr int B_BYTES_N = KS_N * SUB_BN;
  static constexpr int BYTES_W = A_BYTES_W + B_BYTES_W;
  static constexpr int BYTES_N = A_BYTES_N + B_BYTES_N;
  static constexpr int STAGE_BYTES = 64 * 1024;
  static constexpr int STAGES = 3;
  static_assert(BYTES_W <= STAGE_BYTES && BYTES_N <= STAGE_BYTES, "stage contents fit a slot");
  static_assert(STAGE_BYTES % 1024 == 0 && SUB_A % 1024 == 0 && SUB_BN % 1024 == 0 &&
                    SUB_BW % 1024 == 0,
                "swizzle atoms stay aligned");
  static_assert(kPairBN / 2 == kBN, "the wide token-row box is kPairBN / 2 rows");
};

// A tile is narrow when this CTA's token half of it fits one 32-row box.
__device__ __forceinline__ bool narrow_tile(int n_valid) {
  return (((n_valid + 15) & ~15) >> 1) <= kBBoxRows;
}

// D[tmem of both CTAs] (+)= A[both CTAs' smem] * B[both CTAs' smem]^T.
__device__ __forceinline__ void mma_issue_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// The MMAs of one stage: KS K sub-blocks (nsub of them inside K) x 4 K steps
// of 16, unrolled with constant descriptor offsets (the issue loop's own cost
// adds to every MMA's ~100-cycle issue time).  `first`: the tile's first
// stage, whose first MMA overwrites the accumulator.
template <int KS, int SUB_A, int SUB_B>
__device__ __forceinline__ void issue_stage_pair(uint32_t d, uint64_t ad, uint64_t bd,
                                                 uint32_t idesc, int nsub, bool first) {
#pragma unroll
  for (int h = 0; h < KS; ++h) {
    if (h == 0 || h < nsub) {
#pragma unroll
      for (int kk = 0; kk < kBK / 16; ++kk)
        mma_issue_pair(d, ad + static_cast<uint64_t>((h * SUB_A + kk * 32) >> 4),
                       bd + static_cast<uint64_t>((h * SUB_B + kk * 32) >> 4), idesc,
                       (first && h == 0 && kk == 0) ? 0u : 1u);
    }
  }
}

}  // namespace gemm
}  // namespace moe
