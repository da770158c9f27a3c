// Device code of the warp-per-token top-k (K2), shared by the top-k kernels
// (router.cu) and the fused persistent MoE kernel (fused_moe.cu).
//
// The routing order follows sglang-jax issue #1367 "Support Step 3.5 Flash",
// section "Key difficulties", item 1: sigmoid scores in fp32; the router bias
// only selects the top-k; the gating weights are the bias-free scores of the
// selected experts, normalised over the top-k and multiplied by the routed
// scaling factor.
//
// After the tensor-core router (band > 0) the logits are approximations: the
// tensor cores' fp32 accumulation over the H products of each part truncates
// at every step (errors up to ~1e-4 at H = 4096).  They are used only to rule
// experts out.  Every expert whose approximate selection score is within
// `band` of the approximate k-th one -- the approximate top-k included -- is
// a candidate, and the warp recomputes its logit as an fp32 dot product on the
// CUDA cores (the token's bf16 row widened exactly, the expert's fp32 router
// column read as a contiguous row of W_r^T).  The selection, its order and
// the gate weights then come from these fp32 logits; non-candidates are
// excluded, which is exact as long as the tensor-core error in the selection
// score stays below band / 2.
#pragma once

#include <float.h>
#include <math.h>

#include "moe_internal.h"

namespace moe {
namespace topk {

// Unsigned key with the order of the float (no NaN): -0 is taken as +0.
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// The k-th largest of the warp's values (lane l holds v[i] for slot l + 32 i;
// equal values count separately, so it is the k-th selection score of any
// ordering by value), 1 <= k <= the number of slots.  Each round takes one
// largest remaining value: a lane-local maximum, a warp max-reduction of its
// key, and the lowest lane holding it retires one copy.
template <int MPL>
__device__ __forceinline__ float warp_kth_largest(const float (&v)[MPL], int k) {
  const int lane = threadIdx.x & 31;
  uint32_t key[MPL];
#pragma unroll
  for (int i = 0; i < MPL; ++i) key[i] = order_key(v[i]);
  uint32_t taken = 0, best = 0;
  for (int j = 0; j < k; ++j) {
    uint32_t m = 0;  // below every key: a lane with nothing left never wins
    int mi = 0;
#pragma unroll
    for (int i = 0; i < MPL; ++i) {
      const bool better = !((taken >> i) & 1u) && key[i] > m;
      m = better ? key[i] : m;
      mi = better ? i : mi;
    }
    best = __reduce_max_sync(0xffffffffu, m);
    const uint32_t holders = __ballot_sync(0xffffffffu, m == best);
    if (lane == __ffs(holders) - 1) taken |= 1u << mi;
  }
  return key_value(best);
}

// Register arg-max rounds over (selection score, lower index first); lane j < k
// ends with the j-th pick and its bias-free score; every lane gets the k-th
// selection score (kth).
template <int MPL>
__device__ __forceinline__ void warp_select_regs(const float (&sc)[MPL], const float (&be)[MPL],
                                                 int E, int k, int& my_idx, float& my_s,
                                                 float& kth) {
  const int lane = threadIdx.x & 31;
  uint32_t taken = 0;
  my_idx = 0;
  my_s = 0.f;
  kth = -INFINITY;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < MPL; ++i) {
      const int e = lane + 32 * i;
      const bool free_ = !((taken >> i) & 1u) && e < E;
      if (free_ && (be[i] > bv || (be[i] == bv && e < bi))) {
        bv = be[i];
        bi = e;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    kth = bv;
    if (bi >= E) bi = 0;  // only reachable with non-finite scores (unsupported input)
    float s_sel = 0.f;
    if ((bi & 31) == lane) {
      const int ii = bi >> 5;
#pragma unroll
      for (int i = 0; i < MPL; ++i)
        if (i == ii) {
          taken |= 1u << i;
          s_sel = sc[i];
        }
    }
    s_sel = __shfl_sync(0xffffffffu, s_sel, bi & 31);
    if (lane == j) {
      my_idx = bi;
      my_s = s_sel;
    }
  }
}

// fp32 dot product of the token's bf16 row with the expert's fp32 router
// column (a row of W_r^T): lane-strided chunks of four, four partial sums,
// fixed shuffle tree; every lane returns the result.
__device__ __forceinline__ float router_dot(const __nv_bfloat16* __restrict__ xt,
                                            const float* __restrict__ wrow, int H) {
  const int lane = threadIdx.x & 31;
  const float4* w4 = reinterpret_cast<const float4*>(wrow);
  const uint2* x4 = reinterpret_cast<const uint2*>(xt);
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 8
  for (int i = lane; i < H / 4; i += 32) {
    const float4 wv = __ldg(w4 + i);
    const uint2 xq = __ldg(x4 + i);
    const float2 x01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xq.x));
    const float2 x23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xq.y));
    a0 = fmaf(x01.x, wv.x, a0);
    a1 = fmaf(x01.y, wv.y, a1);
    a2 = fmaf(x23.x, wv.z, a2);
    a3 = fmaf(x23.y, wv.w, a3);
  }
  float acc = (a0 + a1) + (a2 + a3);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  return acc;
}

// Two such dot products (experts e0 and e1) with their loads interleaved
// (four iterations' loads in flight: more would cost the registers that let
// more warps run; the order of each partial sum is the same either way).
__device__ __forceinline__ void router_dot2(const __nv_bfloat16* __restrict__ xt,
                                            const float* __restrict__ w0,
                                            const float* __restrict__ w1, int H, float& r0,
                                            float& r1) {
  const int lane = threadIdx.x & 31;
  const float4* p0 = reinterpret_cast<const float4*>(w0);
  const float4* p1 = reinterpret_cast<const float4*>(w1);
  const uint2* x4 = reinterpret_cast<const uint2*>(xt);
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  float b0 = 0.f, b1 = 0.f, b2 = 0.f, b3 = 0.f;
#pragma unroll 4
  for (int i = lane; i < H / 4; i += 32) {
    const float4 u = __ldg(p0 + i);
    const float4 v = __ldg(p1 + i);
    const uint2 xq = __ldg(x4 + i);
    const float2 x01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xq.x));
    const float2 x23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xq.y));
    a0 = fmaf(x01.x, u.x, a0);
    a1 = fmaf(x01.y, u.y, a1);
    a2 = fmaf(x23.x, u.z, a2);
    a3 = fmaf(x23.y, u.w, a3);
    b0 = fmaf(x01.x, v.x, b0);
    b1 = fmaf(x01.y, v.y, b1);
    b2 = fmaf(x23.x, v.z, b2);
    b3 = fmaf(x23.y, v.w, b3);
  }
  float acc = (a0 + a1) + (a2 + a3);
  float bcc = (b0 + b1) + (b2 + b3);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    acc += __shfl_xor_sync(0xffffffffu, acc, off);
    bcc += __shfl_xor_sync(0xffffffffu, bcc, off);
  }
  r0 = acc;
  r1 = bcc;
}

// The warp-per-token top-k of one token t (all 32 lanes of the calling warp):
// sums the ksplit partial logits of each expert (lane l owns experts l, l +
// 32, ...; fixed order), forms the fp32 sigmoid scores and the selection
// scores with s_bias (the router bias, or zeros), selects, and writes the
// token's top-k indices and gate weights (and its logits when logits_out is
// set).  With rf.band > 0 (after the tensor-core router) the approximate
// scores only rule experts out and the candidates are recomputed in fp32 (see
// the comment above).  c_list: this warp's 32 ints of scratch (shared memory).
template <int MPL>
__device__ __forceinline__ void topk_warp_token(int t, const float* __restrict__ partial,
                                                int ksplit, int T, int E, int k,
                                                const float* s_bias, int* c_list, int norm,
                                                float scale, int* __restrict__ topk_idx,
                                                float* __restrict__ topk_w,
                                                float* __restrict__ logits_out,
                                                const TopkRefine& rf) {
  const int lane = threadIdx.x & 31;
  const size_t zstride = static_cast<size_t>(T) * E;
  const float* src = partial + static_cast<size_t>(t) * E + lane;
  // per expert: partial z goes to accumulator z % 4 while four remain, the
  // rest to the first one; (a0 + a1) + (a2 + a3).  The z loop is outermost so
  // the loads of all the lane's experts are in flight together.
  float a0[MPL], a1[MPL], a2[MPL], a3[MPL];
#pragma unroll
  for (int i = 0; i < MPL; ++i) a0[i] = a1[i] = a2[i] = a3[i] = 0.f;
  int z = 0;
  for (; z + 4 <= ksplit; z += 4) {
#pragma unroll
    for (int i = 0; i < MPL; ++i) {
      if (lane + 32 * i < E) {
        a0[i] += src[(z + 0) * zstride + 32 * i];
        a1[i] += src[(z + 1) * zstride + 32 * i];
        a2[i] += src[(z + 2) * zstride + 32 * i];
        a3[i] += src[(z + 3) * zstride + 32 * i];
      }
    }
  }
  for (; z < ksplit; ++z) {
#pragma unroll
    for (int i = 0; i < MPL; ++i)
      if (lane + 32 * i < E) a0[i] += src[z * zstride + 32 * i];
  }
  float l[MPL], sc[MPL], be[MPL];
#pragma unroll
  for (int i = 0; i < MPL; ++i) {
    const int e = lane + 32 * i;
    l[i] = 0.f;
    sc[i] = 0.f;
    be[i] = -INFINITY;
    if (e < E) {
      l[i] = (a0[i] + a1[i]) + (a2[i] + a3[i]);
      sc[i] = 1.0f / (1.0f + expf(-l[i]));
      be[i] = sc[i] + s_bias[e];
    }
  }
  int my_idx = 0;
  float my_s = 0.f, kth;
  if (rf.band > 0.f)
    kth = warp_kth_largest<MPL>(be, k);  // the picks come from the refined scores below
  else
    warp_select_regs<MPL>(sc, be, E, k, my_idx, my_s, kth);
  int c_e = 0x7fffffff;  // after the refinement: lane c's candidate and its fp32 logit
  float c_l = 0.f;
  if (rf.band > 0.f) {
    const float floor_ = kth - rf.band;
    const __nv_bfloat16* xt = rf.x + static_cast<size_t>(t) * rf.H;
    // candidates in expert order, listed in this warp's slice of shared
    // memory (at most 32 recomputed in parallel pairs; more fall back below)
    int n = 0;
#pragma unroll
    for (int i = 0; i < MPL; ++i) {
      const bool cand = be[i] >= floor_ && lane + 32 * i < E;
      const uint32_t m = __ballot_sync(0xffffffffu, cand);
      if (!cand) be[i] = -INFINITY;  // ruled out
      const int at = n + __popc(m & ((1u << lane) - 1u));
      if (cand && at < 32) c_list[at] = lane + 32 * i;
      n += __popc(m);
    }
    __syncwarp();
    const int n_list = n < 32 ? n : 32;
    // lane c keeps candidate c's fp32 logit and scores
    c_e = lane < n_list ? c_list[lane] : 0x7fffffff;
    float c_be = -INFINITY, c_s = 0.f;
    for (int c = 0; c < n_list; c += 2) {
      const int e0 = c_list[c];
      const int e1 = c + 1 < n_list ? c_list[c + 1] : e0;
      float r0, r1;
      router_dot2(xt, rf.w_t + static_cast<size_t>(e0) * rf.H,
                  rf.w_t + static_cast<size_t>(e1) * rf.H, rf.H, r0, r1);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (c + h >= n_list) continue;
        const int e = h == 0 ? e0 : e1;
        const float acc = h == 0 ? r0 : r1;
        const float sv = 1.0f / (1.0f + expf(-acc));
        const float bv = sv + s_bias[e];
        if (lane == c + h) {
          c_l = acc;
          c_be = bv;
          c_s = sv;
        }
      }
    }
    if (n > 32) {
      // rare: hand the first 32 results to their owner lanes, then the
      // candidates past them one at a time (the list is rebuilt from the
      // registers: ruled-out experts are at -inf)
#pragma unroll
      for (int i = 0; i < MPL; ++i)
        for (int c = 0; c < 32; ++c) {
          const int ec = __shfl_sync(0xffffffffu, c_e, c);
          const float lc = __shfl_sync(0xffffffffu, c_l, c);
          const float sc_c = __shfl_sync(0xffffffffu, c_s, c);
          const float bc = __shfl_sync(0xffffffffu, c_be, c);
          if (ec == lane + 32 * i) {
            l[i] = lc;
            sc[i] = sc_c;
            be[i] = bc;
          }
        }
      int seen = 0;
#pragma unroll
      for (int i = 0; i < MPL; ++i) {
        uint32_t m = __ballot_sync(0xffffffffu, be[i] > -INFINITY && lane + 32 * i < E);
        while (m != 0u) {
          const int src_lane = __ffs(m) - 1;
          m &= m - 1u;
          if (seen >= 32) {  // the first 32 are recomputed already
            const int e = src_lane + 32 * i;
            const float acc = router_dot(xt, rf.w_t + static_cast<size_t>(e) * rf.H, rf.H);
            const float sv = 1.0f / (1.0f + expf(-acc));
            if (lane == src_lane) {
              l[i] = acc;
              sc[i] = sv;
              be[i] = sv + s_bias[e];
            }
          }
          ++seen;
        }
      }
    }
    if (n <= 32) {
      // order the candidates by rank: the number of candidates ahead of a
      // candidate (higher score, or equal score and lower index); the lane
      // with rank j supplies the j-th pick
      int rank = 0;
      for (int c = 0; c < n; ++c) {
        const float bc = __shfl_sync(0xffffffffu, c_be, c);
        const int ec = __shfl_sync(0xffffffffu, c_e, c);
        rank += (bc > c_be || (bc == c_be && ec < c_e)) ? 1 : 0;
      }
      int pick_e = 0;
      float pick_s = 0.f;
      for (int c = 0; c < n; ++c) {
        const int rc = __shfl_sync(0xffffffffu, rank, c);
        const int ec = __shfl_sync(0xffffffffu, c_e, c);
        const float s_c = __shfl_sync(0xffffffffu, c_s, c);
        if (rc == lane) {
          pick_e = ec;
          pick_s = s_c;
        }
      }
      my_idx = pick_e;
      my_s = pick_s;
    } else {
      warp_select_regs<MPL>(sc, be, E, k, my_idx, my_s, kth);
    }
  }
  if (logits_out != nullptr) {
    float* lo = logits_out + static_cast<size_t>(t) * E;
#pragma unroll
    for (int i = 0; i < MPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E) lo[e] = l[i];
    }
    __syncwarp();
    if (c_e < E) lo[c_e] = c_l;  // the recomputed logits replace the approximate ones
  }
  float sum = 0.f;
  for (int j = 0; j < k; ++j) sum += __shfl_sync(0xffffffffu, my_s, j);
  if (lane < k) {
    topk_idx[static_cast<size_t>(t) * k + lane] = my_idx;
    topk_w[static_cast<size_t>(t) * k + lane] = norm ? (my_s / sum) * scale : my_s * scale;
  }
}


}  // namespace topk
}  // namespace moe
