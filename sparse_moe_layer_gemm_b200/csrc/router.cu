// K1: router logits l = x . W_r in fp32, and K2: sigmoid scores, top-k on the
// biased scores, bias-free renormalised and scaled gate weights.
//
// The routing order follows sglang-jax issue #1367 "Support Step 3.5 Flash",
// section "Key difficulties", item 1: sigmoid scores in fp32; the router bias
// only selects the top-k; the gating weights are the bias-free scores of the
// selected experts, normalised over the top-k and multiplied by the routed
// scaling factor (llm-atlas "Step-3.5-Flash", "Raw config fields":
// moe_router_activation sigmoid, moe_router_scaling_factor 3,
// norm_expert_weight true, use_moe_router_bias true, need_fp32_gate true).
#include <float.h>
#include <math.h>

#include "moe_internal.h"
#include "moe_ptx.cuh"
#include "topk_warp.cuh"

namespace moe {

namespace {

using topk::order_key;
using topk::router_dot;
using topk::router_dot2;
using topk::warp_kth_largest;
using topk::warp_select_regs;

__device__ __forceinline__ void load8_as_f32(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 q = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

__device__ __forceinline__ void load8_as_f32(const float* p, float (&v)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// One block: kRouterTok tokens x kRouterExp experts over one K slice
// [z * kchunk, (z+1) * kchunk).  256 threads, each 4 tokens x 6 experts
// (experts strided by 16 so a warp reads 16 consecutive weights).  x is
// widened to fp32 exactly; products accumulate in fp32 FMAs.
template <typename TX>
__global__ void __launch_bounds__(256) router_logits_kernel(const TX* __restrict__ x,
                                                            const float* __restrict__ wr,
                                                            float* __restrict__ partial, int T,
                                                            int H, int E, int kchunk) {
  pdl_wait();  // the previous kernel's results are visible
  __shared__ __align__(16) float xs[kRouterKStep][kRouterTok + 4];
  __shared__ __align__(16) float ws[kRouterKStep][kRouterExp];
  const int e0 = blockIdx.x * kRouterExp;
  const int t0 = blockIdx.y * kRouterTok;
  const int z = blockIdx.z;
  const int kbeg = z * kchunk;
  const int kend = min(H, kbeg + kchunk);
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;

  float acc[4][6];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 6; ++j) acc[i][j] = 0.f;

  for (int k0 = kbeg; k0 < kend; k0 += kRouterKStep) {
    {  // x tile: 64 tokens x 32 k, 8 consecutive k per thread, stored k-major
      const int tl = tid >> 2, kq = (tid & 3) * 8;
      const int t = t0 + tl;
      float v[8];
      if (t < T) {
        load8_as_f32(x + static_cast<size_t>(t) * H + k0 + kq, v);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) xs[kq + i][tl] = v[i];
    }
    for (int i = tid; i < kRouterKStep * kRouterExp; i += 256) {  // W tile: 32 k x 96 experts
      const int kk = i / kRouterExp, ee = i % kRouterExp;
      const int e = e0 + ee;
      ws[kk][ee] = (e < E) ? wr[static_cast<size_t>(k0 + kk) * E + e] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kRouterKStep; ++kk) {
      const float4 xv = *reinterpret_cast<const float4*>(&xs[kk][ty * 4]);
      const float xa[4] = {xv.x, xv.y, xv.z, xv.w};
      float wv[6];
#pragma unroll
      for (int j = 0; j < 6; ++j) wv[j] = ws[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 6; ++j) acc[i][j] = fmaf(xa[i], wv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = t0 + ty * 4 + i;
    if (t >= T) continue;
#pragma unroll
    for (int j = 0; j < 6; ++j) {
      const int e = e0 + tx + 16 * j;
      if (e < E) partial[(static_cast<size_t>(z) * T + t) * E + e] = acc[i][j];
    }
  }
}

// k rounds of a warp arg-max on (selection score, lower index first) over the
// scores in shared memory: lane l holds experts l, l + 32, ... (MPL per lane);
// the owner lane hands over the bias-free score of the winner.  Lane j < k
// ends with the j-th pick; every lane gets the k-th selection score (kth) and
// the best remaining one after k picks (next, -inf when k == E).
template <int MPL>
__device__ __forceinline__ void warp_select(const float* s_sc, const float* s_be, int E, int k,
                                            int& my_idx, float& my_s, float& kth, float& next) {
  const int lane = threadIdx.x & 31;
  float sc[MPL], be[MPL];
#pragma unroll
  for (int i = 0; i < MPL; ++i) {
    const int e = lane + 32 * i;
    sc[i] = (e < E) ? s_sc[e] : 0.f;
    be[i] = (e < E) ? s_be[e] : -INFINITY;
  }
  uint32_t taken = 0;
  my_idx = 0;
  my_s = 0.f;
  kth = -INFINITY;
  next = -INFINITY;
  for (int j = 0; j <= k; ++j) {
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
    if (j == k) {  // the best score left after the k picks
      next = bv;
      break;
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

// Block-per-token form (small and medium batches: more threads per token,
// so the latency of one token's work is shorter).  Thread e sums the ksplit partial logits of expert e
// (independent loads, fixed order), forms the fp32 sigmoid score s and the
// selection score s + b in shared memory; warp 0 selects.
//
// After the tensor-core router (band > 0) the logits are approximations: the
// tensor cores' fp32 accumulation over the 3H products truncates at every
// step (errors up to ~1e-4 at H = 4096).  They are used only to rule experts
// out.  Every expert whose approximate selection score is within `band` of
// the approximate k-th one -- the approximate top-k included -- is a
// candidate; one warp per candidate recomputes its logit as an fp32 dot
// product on the CUDA cores (the token's row staged in shared memory, the
// expert's fp32 router column read as a contiguous row of W_r^T).  The selection, its order and the gate weights then come from these
// fp32 logits; non-candidates are excluded, which is exact as long as the
// tensor-core error in the selection score stays below band / 2.
template <int MPL>
__global__ void __launch_bounds__(1024) topk_block_kernel(const float* __restrict__ partial, int ksplit,
                                                    int T, int E, int k,
                                                    const float* __restrict__ bias, int norm,
                                                    float scale, int* __restrict__ topk_idx,
                                                    float* __restrict__ topk_w,
                                                    float* __restrict__ logits_out,
                                                    TopkRefine rf) {
  pdl_wait();  // the previous kernel's results are visible
  __shared__ float s_l[32 * MPL];
  __shared__ float s_sc[32 * MPL];
  __shared__ float s_be[32 * MPL];
  __shared__ int s_cand[32 * MPL];
  __shared__ float s_cb[32];     // selection scores of the first 32 candidates
  __shared__ int s_rank_e[32];   // the candidates by rank
  __shared__ int s_ncand;
  __shared__ float s_kth;
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const float* src = partial + static_cast<size_t>(t) * E + e;
    const size_t zstride = static_cast<size_t>(T) * E;
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    int z = 0;
    for (; z + 4 <= ksplit; z += 4) {
      a0 += src[(z + 0) * zstride];
      a1 += src[(z + 1) * zstride];
      a2 += src[(z + 2) * zstride];
      a3 += src[(z + 3) * zstride];
    }
    for (; z < ksplit; ++z) a0 += src[z * zstride];
    const float l = (a0 + a1) + (a2 + a3);
    const float s = 1.0f / (1.0f + expf(-l));
    s_l[e] = l;
    s_sc[e] = s;
    s_be[e] = (bias != nullptr) ? s + bias[e] : s;
  }
  __syncthreads();
  int my_idx = 0;
  float my_s = 0.f, kth, next;
  if (rf.band > 0.f) {
    if (warp == 0) {  // only the k-th approximate selection score is needed here
      float v[MPL];
#pragma unroll
      for (int i = 0; i < MPL; ++i) v[i] = lane + 32 * i < E ? s_be[lane + 32 * i] : -INFINITY;
      const float kth_approx = warp_kth_largest<MPL>(v, k);
      if (lane == 0) {
        s_kth = kth_approx;
        s_ncand = 0;
      }
    }
    // the token's input row, widened to fp32 once for all candidate warps
    extern __shared__ float s_x[];
    const int H = rf.H;
    const __nv_bfloat16* xt = rf.x + static_cast<size_t>(t) * H;
    for (int h = threadIdx.x * 8; h < H; h += blockDim.x * 8) {
      const uint4 q = *reinterpret_cast<const uint4*>(xt + h);
      const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(hv[i]);
        s_x[h + 2 * i] = f.x;
        s_x[h + 2 * i + 1] = f.y;
      }
    }
    __syncthreads();
    const float floor_ = s_kth - rf.band;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      if (s_be[e] >= floor_)
        s_cand[atomicAdd(&s_ncand, 1)] = e;
      else
        s_be[e] = -INFINITY;  // ruled out
    }
    __syncthreads();
    const int n = s_ncand;
    for (int c = warp; c < n; c += nwarps) {
      // fp32 dot product with the expert's router column (a row of W_r^T):
      // lane-strided float4 chunks, four partial sums, fixed shuffle tree
      const int e = s_cand[c];
      const float4* w4 = reinterpret_cast<const float4*>(rf.w_t + static_cast<size_t>(e) * H);
      const float4* x4 = reinterpret_cast<const float4*>(s_x);
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll 8
      for (int i = lane; i < H / 4; i += 32) {
        const float4 wv = __ldg(w4 + i);
        const float4 xv = x4[i];
        a0 = fmaf(xv.x, wv.x, a0);
        a1 = fmaf(xv.y, wv.y, a1);
        a2 = fmaf(xv.z, wv.z, a2);
        a3 = fmaf(xv.w, wv.w, a3);
      }
      float acc = (a0 + a1) + (a2 + a3);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (lane == 0) {
        const float sv = 1.0f / (1.0f + expf(-acc));
        s_l[e] = acc;
        s_sc[e] = sv;
        s_be[e] = (bias != nullptr) ? sv + bias[e] : sv;
      }
    }
    __syncthreads();
    if (n <= 32) {
      // order the candidates by rank: lane c holds candidate c; its rank is
      // the number of candidates ahead of it (higher score, or equal score
      // and lower index); the lane with rank j supplies the j-th pick.  The
      // candidates' scores are listed beside them so the rank loop's loads
      // are independent.
      if (warp == 0) {
        const int e = lane < n ? s_cand[lane] : 0x7fffffff;
        const float b = lane < n ? s_be[e] : -INFINITY;
        if (lane < n) s_cb[lane] = b;
        __syncwarp();
        int rank = 0;
#pragma unroll 4
        for (int c = 0; c < n; ++c) {
          const float bc = s_cb[c];
          const int ec = s_cand[c];
          rank += (bc > b || (bc == b && ec < e)) ? 1 : 0;
        }
        if (lane < n) s_rank_e[rank] = e;  // ranks are distinct
        __syncwarp();
        my_idx = lane < n ? s_rank_e[lane] : 0;
        my_s = lane < n ? s_sc[my_idx] : 0.f;
      }
    } else if (warp == 0) {
      warp_select<MPL>(s_sc, s_be, E, k, my_idx, my_s, kth, next);
    }
  } else if (warp == 0) {
    warp_select<MPL>(s_sc, s_be, E, k, my_idx, my_s, kth, next);
  }
  if (logits_out != nullptr) {
    for (int e = threadIdx.x; e < E; e += blockDim.x)
      logits_out[static_cast<size_t>(t) * E + e] = s_l[e];
  }
  if (warp != 0) return;
  float sum = 0.f;
  for (int j = 0; j < k; ++j) sum += __shfl_sync(0xffffffffu, my_s, j);
  if (lane < k) {
    topk_idx[static_cast<size_t>(t) * k + lane] = my_idx;
    topk_w[static_cast<size_t>(t) * k + lane] = norm ? (my_s / sum) * scale : my_s * scale;
  }
}

// Warp-per-token form (large batches).  One warp per token (up to kTopkWarps
// tokens per block); the per-token work (topk_warp_token, topk_warp.cuh):
// lane l owns experts l, l + 32, ... (MPL per lane), sums their ksplit
// partial logits (independent loads, fixed order), forms the fp32 sigmoid
// score s and the selection score s + b in registers; the warp then selects,
// recomputing the boundary candidates in fp32 after the tensor-core router.
constexpr int kTopkWarps = 8;
// Token count from which the warp-per-token form runs (both forms give the
// same bits).  Measured at 4096 tokens (288 experts, tensor-core router):
// 0.063 ms against the block form's 0.088.
constexpr int kTopkWarpMinTokens = 2048;

// Four blocks (32 warps) per SM: the candidate recomputation is bound by L2
// latency, so warps in flight matter more than registers (64 a thread, a few
// spilled; at 80 registers only three blocks fit and the Zipf top-k took
// 0.284 ms instead of 0.201).
template <int MPL>
__global__ void __launch_bounds__(32 * kTopkWarps, 4) topk_warp_kernel(
    const float* __restrict__ partial, int ksplit, int T, int E, int k,
    const float* __restrict__ bias, int norm, float scale, int* __restrict__ topk_idx,
    float* __restrict__ topk_w, float* __restrict__ logits_out, TopkRefine rf) {
  pdl_wait();  // the previous kernel's results are visible
  extern __shared__ float s_bias[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_bias[e] = bias != nullptr ? bias[e] : 0.f;
  __syncthreads();
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  int* c_list = reinterpret_cast<int*>(s_bias + E) + (threadIdx.x >> 5) * 32;
  topk::topk_warp_token<MPL>(t, partial, ksplit, T, E, k, s_bias, c_list, norm, scale, topk_idx,
                             topk_w, logits_out, rf);
}

}  // namespace

cudaError_t launch_router_logits(const void* x, bool x_bf16, const float* router_w, float* partial,
                                 int T, int H, int E, int ksplit, cudaStream_t st) {
  const int kchunk = H / ksplit;
  dim3 grid((E + kRouterExp - 1) / kRouterExp, (T + kRouterTok - 1) / kRouterTok, ksplit);
  if (x_bf16)
    return launch_pdl(router_logits_kernel<__nv_bfloat16>, grid, dim3(256), 0, st,
                      static_cast<const __nv_bfloat16*>(x), router_w, partial, T, H, E, kchunk);
  return launch_pdl(router_logits_kernel<float>, grid, dim3(256), 0, st,
                    static_cast<const float*>(x), router_w, partial, T, H, E, kchunk);
}

cudaError_t topk_configure_device() {
  // dynamic shared memory of the block form's candidate recomputation: one
  // fp32 input row
  const int bytes = 16384 * static_cast<int>(sizeof(float));
  cudaError_t e = cudaSuccess;
#define MOE_TOPK_ATTR(N)                                                                       \
  if (e == cudaSuccess)                                                                        \
    e = cudaFuncSetAttribute(topk_block_kernel<N>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             bytes);
  MOE_TOPK_ATTR(1) MOE_TOPK_ATTR(2) MOE_TOPK_ATTR(4) MOE_TOPK_ATTR(8) MOE_TOPK_ATTR(9)
  MOE_TOPK_ATTR(16) MOE_TOPK_ATTR(32)
#undef MOE_TOPK_ATTR
  return e;
}

cudaError_t launch_topk(const float* partial, int ksplit, int T, int E, int k, const float* bias,
                        bool norm, float scale, int* topk_idx, float* topk_w, cudaStream_t st,
                        float* logits_out, const TopkRefine* refine) {
  const int mpl = (E + 31) / 32;
  TopkRefine rf{};
  if (refine != nullptr) rf = *refine;
  if (T < kTopkWarpMinTokens) {
    const int threads = min(1024, max(32, (E + 31) / 32 * 32));
    const size_t smem = rf.band > 0.f ? static_cast<size_t>(rf.H) * sizeof(float) : 0;
#define MOE_TOPK(N)                                                                        \
  return launch_pdl(topk_block_kernel<N>, dim3(T), dim3(threads), smem, st, partial, ksplit, T, E, \
                    k, bias, norm ? 1 : 0, scale, topk_idx, topk_w, logits_out, rf)
    if (mpl <= 1) MOE_TOPK(1);
    else if (mpl <= 2) MOE_TOPK(2);
    else if (mpl <= 4) MOE_TOPK(4);
    else if (mpl <= 8) MOE_TOPK(8);
    else if (mpl <= 9) MOE_TOPK(9);
    else if (mpl <= 16) MOE_TOPK(16);
    else MOE_TOPK(32);
#undef MOE_TOPK
    return cudaGetLastError();
  }
  const int blocks = (T + kTopkWarps - 1) / kTopkWarps;
  // router bias, then per warp a list of up to 32 candidates
  const size_t smem = static_cast<size_t>(E) * sizeof(float) + kTopkWarps * 32 * sizeof(int);
#define MOE_TOPK(N)                                                                            \
  return launch_pdl(topk_warp_kernel<N>, dim3(blocks), dim3(32 * kTopkWarps), smem, st, partial,   \
                    ksplit, T, E, k, bias, norm ? 1 : 0, scale, topk_idx, topk_w, logits_out, rf)
  if (mpl <= 1) MOE_TOPK(1);
  else if (mpl <= 2) MOE_TOPK(2);
  else if (mpl <= 4) MOE_TOPK(4);
  else if (mpl <= 8) MOE_TOPK(8);
  else if (mpl <= 9) MOE_TOPK(9);
  else if (mpl <= 16) MOE_TOPK(16);
  else MOE_TOPK(32);
#undef MOE_TOPK
  return cudaGetLastError();
}

}  // namespace moe
