// Device code of the weighted combine (K7), shared by the combine kernel
// (combine.cu) and the fused persistent MoE kernel (fused_moe.cu):
// out[t] = sum_j y[pos(t, j)] + y[shared row t], summed in fp32 in the fixed
// order j = 0..k-1 then the shared row, rounded once to the output dtype.
#pragma once

#include <cuda_bf16.h>

namespace moe {
namespace combine {

__device__ __forceinline__ void add8(float (&acc)[8], const __nv_bfloat16* p) {
  const uint4 q = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    acc[2 * i] += f.x;
    acc[2 * i + 1] += f.y;
  }
}

// fp32 rows (the fp32 expert path)
__device__ __forceinline__ void add8(float (&acc)[8], const float* p) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  acc[0] += a.x;
  acc[1] += a.y;
  acc[2] += a.z;
  acc[3] += a.w;
  acc[4] += b.x;
  acc[5] += b.y;
  acc[6] += b.z;
  acc[7] += b.w;
}

// acc += the 8 bf16 values held in q (already loaded)
__device__ __forceinline__ void add8(float (&acc)[8], const uint4& q) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    acc[2 * i] += f.x;
    acc[2 * i + 1] += f.y;
  }
}

// 8 consecutive values of a y row, as loaded (bf16: one 16-byte vector;
// fp32: two)
struct Row8F32 {
  float4 a, b;
};
template <typename TY>
struct Row8;
template <>
struct Row8<__nv_bfloat16> {
  using type = uint4;
};
template <>
struct Row8<float> {
  using type = Row8F32;
};

__device__ __forceinline__ uint4 load8(const __nv_bfloat16* p) {
  return *reinterpret_cast<const uint4*>(p);
}
__device__ __forceinline__ Row8F32 load8(const float* p) {
  return Row8F32{*reinterpret_cast<const float4*>(p), *reinterpret_cast<const float4*>(p + 4)};
}
__device__ __forceinline__ void add8(float (&acc)[8], const Row8F32& q) {
  acc[0] += q.a.x;
  acc[1] += q.a.y;
  acc[2] += q.a.z;
  acc[3] += q.a.w;
  acc[4] += q.b.x;
  acc[5] += q.b.y;
  acc[6] += q.b.z;
  acc[7] += q.b.w;
}

// Rows a combine thread loads at once (k + 1 <= kPreRows: every row's vector
// in flight together, then the sum in the fixed order).
constexpr int kPreRows = 9;

__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&v)[8]) {
  uint4 q;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&q);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = q;
}

__device__ __forceinline__ void store8(float* p, const float (&v)[8]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}

// Token t's output row, by all threads of the block (threadIdx.x / blockDim.x
// strides over the row's 8-element vectors); rows_s: k + 1 ints of shared
// memory.  Ends with a __syncthreads, so rows_s may be reused at once.
template <typename TO, typename TY>
__device__ __forceinline__ void combine_token(int t, const TY* __restrict__ y,
                                              const int* __restrict__ pos, int T, int k, int H,
                                              int with_shared, TO* __restrict__ out, int* rows_s) {
  if (threadIdx.x < k) rows_s[threadIdx.x] = pos[static_cast<size_t>(t) * k + threadIdx.x];
  if (threadIdx.x == 0) rows_s[k] = with_shared ? T * k + t : -1;
  __syncthreads();
  const int nvec = H / 8;
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    // (row -1: another shard's expert, or no shared expert here)
    if (k + 1 <= kPreRows) {
      // all rows' loads in flight at once (a latency-bound gather otherwise),
      // then added in the same order j = 0..k
      typename Row8<TY>::type q[kPreRows];
#pragma unroll
      for (int j = 0; j < kPreRows; ++j)
        if (j <= k && rows_s[j] >= 0) q[j] = load8(y + static_cast<size_t>(rows_s[j]) * H + v * 8);
#pragma unroll
      for (int j = 0; j < kPreRows; ++j)
        if (j <= k && rows_s[j] >= 0) add8(acc, q[j]);
    } else {
      for (int j = 0; j <= k; ++j)
        if (rows_s[j] >= 0) add8(acc, y + static_cast<size_t>(rows_s[j]) * H + v * 8);
    }
    store8(out + static_cast<size_t>(t) * H + v * 8, acc);
  }
  __syncthreads();
}

}  // namespace combine
}  // namespace moe
