// Weight packing at load time: the caller's x . W layouts become the K-major
// bf16 operands of the grouped GEMMs.
//   gate / up  [G][H][I]  ->  rows g * 2*I_pad + (f / 128) * 256 + half * 128 + f % 128,
//                             columns h (ld H): each 256-row block holds 128 gate
//                             rows then the 128 matching up rows.
//   down       [G][I][H]  ->  rows g * H + n, columns i (ld I_pad).
// Rows and columns past I (up to I_pad, a multiple of 128) stay zero, so the
// padded features compute silu(0) * 0 = 0 and add nothing in the down GEMM.
// fp32 weights (the fp32 expert path) keep the same rows as fp32 [hi | lo]
// halves of the tf32 split (tf32.cuh): column k of the row at k (hi) and at
// K + k (lo), K = H (gate|up) or I_pad (down).
// FP8 E4M3 weights use the same packed rows, one byte per code, with one fp32
// scale per packed row (the row's output feature; zero for padded rows), but
// stored tile-major for the FP8 GEMM: for each tile of TR packed rows (the
// GEMM's weight rows per tile) and each 128-wide K slice (one pipeline
// stage), one contiguous TR x 128 run, ordered (64-code half h, 128-row block
// b, row r, code): byte ((tile * K / 128 + k / 128) * TR * 128 + h * TR * 64
// + b * 8192 + r * 64 + chunk position * 16 + k % 16).  Inside a row the
// 16-code chunk c sits at position c ^ ((r / 2) % 4) (a 64-byte swizzle), so
// that a warp reading one chunk of 32 consecutive rows hits every
// shared-memory bank evenly.  A pipeline stage then reads one contiguous
// TR x 128-byte run with one bulk copy instead of 64-byte pieces of rows
// K bytes apart.
#include "fp8.cuh"
#include "moe_internal.h"
#include "tf32.cuh"

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

// pack_kernel's transpose and rows for the fp32 path: dst rows of 2 * dst_ld
// fp32, the tf32 split's hi half then its lo half.
template <typename TS, bool GU>
__global__ void __launch_bounds__(256) pack_split_kernel(const TS* __restrict__ src, int R, int C,
                                                         float* __restrict__ dst, int dst_ld,
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
      float hi, lo;
      tf32_split(tile[threadIdx.x][i], hi, lo);
      float* row = dst + drow * 2 * static_cast<size_t>(dst_ld);
      row[r] = hi;
      row[dst_ld + r] = lo;
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

// Byte offset of packed row `row`, reduction index k, in the tile-major FP8
// layout (K codes per packed row, tiles of TR rows).
__device__ __forceinline__ size_t fp8_tiled_offset(size_t row, int k, int K, int TR) {
  const size_t tile = row / TR;
  const int rt = static_cast<int>(row % TR), b = rt / 128, r = rt % 128;
  const int h = (k % 128) / 64, kk = k % 64;
  return (tile * (K / 128) + k / 128) * static_cast<size_t>(TR) * 128 +
         static_cast<size_t>(h) * TR * 64 + b * 8192 + r * 64 +
         ((((kk >> 4) ^ ((r >> 1) & 3))) << 4) + (kk & 15);
}

// Byte transpose of the [R][C] code matrix of group blockIdx.z (FP8 weights),
// rows placed as in pack_kernel, bytes in the tile-major layout (K = dst_ld,
// tiles of TR rows).
template <bool GU>
__global__ void __launch_bounds__(256) pack_codes_kernel(const uint8_t* __restrict__ src, int R,
                                                         int C, uint8_t* __restrict__ dst,
                                                         int dst_ld, int I_pad, int H, int half,
                                                         int TR) {
  __shared__ uint8_t tile[32][33];
  const int g = blockIdx.z;
  const uint8_t* s = src + static_cast<size_t>(g) * R * C;
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    tile[i][threadIdx.x] = (r < R && c < C) ? s[static_cast<size_t>(r) * C + c] : 0;
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
      dst[fp8_tiled_offset(drow, r, dst_ld, TR)] = tile[threadIdx.x][i];
    }
  }
}

// gate / up scales [G][I] -> the packed gate|up rows' scales.
__global__ void pack_gate_up_scales_kernel(const float* __restrict__ s, int groups, int I,
                                           int I_pad, int half, float* __restrict__ dst) {
  const size_t n = static_cast<size_t>(groups) * I;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int g = static_cast<int>(i / I), f = static_cast<int>(i % I);
    dst[static_cast<size_t>(g) * 2 * I_pad + (f / 128) * 256 + half * 128 + (f % 128)] = s[i];
  }
}

// E4M3 codes -> bf16 through the expert GEMMs' converter routine (4 codes per
// thread step; n % 4 == 0).
__global__ void decode_e4m3_kernel(const uint32_t* __restrict__ codes, size_t n4,
                                   uint2* __restrict__ out) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    uint2 o;
    e4m3x4_to_bf16x4(codes[i], o.x, o.y);
    out[i] = o;
  }
}

}  // namespace

cudaError_t launch_pack_codes_gate_up(const uint8_t* w, int groups, int H, int I, int I_pad,
                                      int half, uint8_t* dst, cudaStream_t st) {
  dim3 grid((I + 31) / 32, (H + 31) / 32, groups), block(32, 8);
  pack_codes_kernel<true><<<grid, block, 0, st>>>(w, H, I, dst, H, I_pad, H, half, 256);
  return cudaGetLastError();
}

cudaError_t launch_pack_codes_down(const uint8_t* w, int groups, int H, int I, int I_pad,
                                   int tile_rows, uint8_t* dst, cudaStream_t st) {
  dim3 grid((H + 31) / 32, (I + 31) / 32, groups), block(32, 8);
  pack_codes_kernel<false><<<grid, block, 0, st>>>(w, I, H, dst, I_pad, I_pad, H, 0, tile_rows);
  return cudaGetLastError();
}

cudaError_t launch_pack_gate_up_scales(const float* s, int groups, int I, int I_pad, int half,
                                       float* dst, cudaStream_t st) {
  pack_gate_up_scales_kernel<<<(groups * I + 255) / 256 < 1024 ? (groups * I + 255) / 256 : 1024,
                               256, 0, st>>>(s, groups, I, I_pad, half, dst);
  return cudaGetLastError();
}

cudaError_t launch_decode_e4m3(const uint8_t* codes, size_t n, __nv_bfloat16* out,
                               cudaStream_t st) {
  const size_t n4 = n / 4;
  const size_t blocks = (n4 + 255) / 256;
  decode_e4m3_kernel<<<static_cast<unsigned>(blocks < 4096 ? (blocks > 0 ? blocks : 1) : 4096),
                       256, 0, st>>>(reinterpret_cast<const uint32_t*>(codes), n4,
                                     reinterpret_cast<uint2*>(out));
  return cudaGetLastError();
}

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

cudaError_t launch_pack_gate_up_split(const void* w, bool w_bf16, int groups, int H, int I,
                                      int I_pad, int half, float* dst, cudaStream_t st) {
  dim3 grid((I + 31) / 32, (H + 31) / 32, groups), block(32, 8);
  if (w_bf16)
    pack_split_kernel<__nv_bfloat16, true><<<grid, block, 0, st>>>(
        static_cast<const __nv_bfloat16*>(w), H, I, dst, H, I_pad, H, half);
  else
    pack_split_kernel<float, true><<<grid, block, 0, st>>>(static_cast<const float*>(w), H, I,
                                                           dst, H, I_pad, H, half);
  return cudaGetLastError();
}

cudaError_t launch_pack_down_split(const void* w, bool w_bf16, int groups, int H, int I,
                                   int I_pad, float* dst, cudaStream_t st) {
  dim3 grid((H + 31) / 32, (I + 31) / 32, groups), block(32, 8);
  if (w_bf16)
    pack_split_kernel<__nv_bfloat16, false><<<grid, block, 0, st>>>(
        static_cast<const __nv_bfloat16*>(w), I, H, dst, I_pad, I_pad, H, 0);
  else
    pack_split_kernel<float, false><<<grid, block, 0, st>>>(static_cast<const float*>(w), I, H,
                                                            dst, I_pad, I_pad, H, 0);
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
