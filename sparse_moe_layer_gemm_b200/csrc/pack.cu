// Weight packing at load time: the caller's x . W layouts become the K-major
// bf16 operands of the grouped GEMMs.
//   gate / up  [G][H][I]  ->  rows g * 2*I_pad + (f / 128) * 256 + half * 128 + f % 128,
//                             columns h (ld H): each 256-row block holds 128 gate
//                             rows then the 128 matching up rows.
//   down       [G][I][H]  ->  rows g * H + n, columns i (ld I_pad).
// Rows and columns past I (up to I_pad, a multiple of 128) stay zero, so the
// padded features compute silu(0) * 0 = 0 and add nothing in the down GEMM.
#include "moe_internal.h"

namespace moe {

namespace {

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

// Transposes the [R][C] matrix of group blockIdx.z through a 32 x 32 tile.
template <typename TS, bool GU>
__global__ void __launch_bounds__(256) pack_kernel(const TS* __restrict__ src, int R, int C,
                                                   __nv_bfloat16* __restrict__ dst, int dst_ld,
                                                   int I_pad, int H, int half) {
  __shared__ float tile[32][33];
  const int g = blockIdx.z;
  const TS* s = src + static_cast<size_t>(g) * R * C;
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    tile[i][threadIdx.x] = (r < R && c < C) ? to_f32(s[static_cast<size_t>(r) * C + c]) : 0.f;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (c < C && r < R) {
      size_t drow;
      if (GU)
        drow = static_cast<size_t>(g) * 2 * I_pad + (c / 128) * 256 + half * 128 + (c % 128);
      else
        drow = static_cast<size_t>(g) * H + c;
      dst[drow * dst_ld + r] = __float2bfloat16_rn(tile[threadIdx.x][i]);
    }
  }
}

// Router weight [H][E] fp32 -> [E_pad][3H] bf16: row e holds W1 | W2 | W3
// along K, with W1 = bf16(w), W2 = bf16(w - W1), W3 = bf16(w - W1 - W2).
// Each residual is exact in fp32 (it keeps at most 16, then 8, significant
// bits), and W3 holds the last 8, so W1 + W2 + W3 == w for normal w.  Rows
// e >= E are zero.  Also writes the fp32 transpose [E][H] (dst_t).
__global__ void __launch_bounds__(256) pack_router_kernel(const float* __restrict__ w, int H, int E,
                                                          int E_pad,
                                                          __nv_bfloat16* __restrict__ dst,
                                                          float* __restrict__ dst_t) {
  __shared__ float tile[32][33];
  const int e0 = blockIdx.x * 32, h0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int h = h0 + i, e = e0 + threadIdx.x;
    tile[i][threadIdx.x] = (h < H && e < E) ? w[static_cast<size_t>(h) * E + e] : 0.f;
  }
  __syncthreads();
  const size_t ld = static_cast<size_t>(3) * H;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int e = e0 + i, h = h0 + threadIdx.x;
    if (e < E_pad && h < H) {
      const float v = tile[threadIdx.x][i];
      const __nv_bfloat16 b1 = __float2bfloat16_rn(v);
      const float r1 = v - __bfloat162float(b1);
      const __nv_bfloat16 b2 = __float2bfloat16_rn(r1);
      const float r2 = r1 - __bfloat162float(b2);
      const __nv_bfloat16 b3 = __float2bfloat16_rn(r2);
      __nv_bfloat16* row = dst + static_cast<size_t>(e) * ld;
      row[h] = b1;
      row[H + h] = b2;
      row[2 * H + h] = b3;
      if (e < E) dst_t[static_cast<size_t>(e) * H + h] = v;
    }
  }
}

}  // namespace

cudaError_t launch_pack_router(const float* w, int H, int E, int E_pad, __nv_bfloat16* dst,
                               float* dst_t, cudaStream_t st) {
  dim3 grid((E_pad + 31) / 32, (H + 31) / 32), block(32, 8);
  pack_router_kernel<<<grid, block, 0, st>>>(w, H, E, E_pad, dst, dst_t);
  return cudaGetLastError();
}

cudaError_t launch_pack_gate_up(const void* w, bool w_bf16, int groups, int H, int I, int I_pad,
                                int half, __nv_bfloat16* dst, cudaStream_t st) {
  dim3 grid((I + 31) / 32, (H + 31) / 32, groups), block(32, 8);
  if (w_bf16)
    pack_kernel<__nv_bfloat16, true><<<grid, block, 0, st>>>(
        static_cast<const __nv_bfloat16*>(w), H, I, dst, H, I_pad, H, half);
  else
    pack_kernel<float, true><<<grid, block, 0, st>>>(static_cast<const float*>(w), H, I, dst, H,
                                                     I_pad, H, half);
  return cudaGetLastError();
}

cudaError_t launch_pack_down(const void* w, bool w_bf16, int groups, int H, int I, int I_pad,
                             __nv_bfloat16* dst, cudaStream_t st) {
  dim3 grid((H + 31) / 32, (I + 31) / 32, groups), block(32, 8);
  if (w_bf16)
    pack_kernel<__nv_bfloat16, false><<<grid, block, 0, st>>>(
        static_cast<const __nv_bfloat16*>(w), I, H, dst, I_pad, I_pad, H, 0);
  else
    pack_kernel<float, false><<<grid, block, 0, st>>>(static_cast<const float*>(w), I, H, dst,
                                                      I_pad, I_pad, H, 0);
  return cudaGetLastError();
}

}  // namespace moe
