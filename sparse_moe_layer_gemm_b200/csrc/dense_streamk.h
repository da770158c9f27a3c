// Interfaces of the dense MLP's one-launch stream-K forward
// (dense_streamk.cu) for its host side (dense_api.cu).  Not installed, not
// part of the ABI.
#pragma once

#include "moe_internal.h"

namespace moe {

// The dense MLP's one-launch stream-K forward (dense_streamk.cu) for up to
// kSkMaxTokens tokens (H % 256 == 0).  2 kSkGroups passes, each split into
// equal per-SM shares of (weight tile, K block) units with fp32 partials per
// segment: gate|up over kSkGroups groups of the 128-feature h tiles, then
// down over the K blocks of the same groups of h, in the same order.
constexpr int kSkMaxTokens = 128;
constexpr int kSkMaxGrid = 200;  // bound of the per-CTA unit tables in shared memory
// (measured at the model's decode size, 64 tokens: one group 0.064 ms, two
// 0.067, three 0.074 -- more passes mean more segments and partials)
constexpr int kSkGroups = 1;
constexpr int kSkPasses = 2 * kSkGroups;

struct SkPass {
  int gemm;          // 0 gate|up, 1 down
  int tile0, tiles;  // its weight tiles (256 rows each)
  int kb0, nkb;      // its K blocks (64 deep) of every tile
};

// The passes for hidden size H and padded intermediate I_pad.  Group g of
// the h tiles is [e_g, e_{g+1}); down pass g reads exactly those h tiles
// (K blocks 2 e_g .. 2 e_{g+1}).
inline void dense_streamk_passes(int H, int I_pad, SkPass (&ps)[kSkPasses]) {
  const int ta = I_pad / 128, tb = H / 256;
  int e[kSkGroups + 1];
  for (int g = 0; g <= kSkGroups; ++g) e[g] = ta * g / kSkGroups;
  for (int g = 0; g < kSkGroups; ++g) {
    ps[g] = SkPass{0, e[g], e[g + 1] - e[g], 0, H / 64};
    ps[kSkGroups + g] = SkPass{1, 0, tb, 2 * e[g], 2 * (e[g + 1] - e[g])};
  }
}

// Counter words of the stream-K forward: the stored segments per tile of
// each pass, the reduced rows per 128-feature tile of h, then three words the
// kernel keeps itself (forwards completed, the sum of their T, CTAs done with
// the current forward), from which every forward derives its targets.
inline int dense_streamk_counters(int H, int I_pad) {
  return 2 * (I_pad / 128) + kSkGroups * (H / 256) + 3;
}

struct DenseStreamK {
  // A operands: packed gate|up [2 I_pad, H] and down [H, I_pad], boxes of
  // 64 x 128 rows; B operands: x [T, H] and h [T, I_pad] (bf16), boxes of
  // 64 x round_up(T, 16) rows
  CUtensorMap tm_gu, tm_dn, tm_x, tm_h;
  int T, H, I_pad;
  int max_seg[kSkPasses];   // dense_streamk_max_seg of each pass
  float limit;
  float* parts[kSkPasses];  // [grid][max_seg][T][256] fp32 per pass
  __nv_bfloat16* h;         // [T, I_pad]
  void* out;                // [T, H], bf16 or fp32
  bool out_f32;
  unsigned int* counters;   // the layer's dense_streamk_counters words (zero at creation
                            // and after a device error)
  int* status;
};

// Segments (tiles touched) of the busiest CTA when `tiles` x `nkb` units are
// split evenly over `grid` CTAs (0 for no units).
int dense_streamk_max_seg(int tiles, int nkb, int grid);
cudaError_t dense_streamk_configure_device(int num_sms);
int dense_streamk_grid();  // 0 before configuration
cudaError_t launch_dense_streamk(const DenseStreamK& d, cudaStream_t st);

}  // namespace moe
