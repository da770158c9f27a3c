// K7: weighted combine.  out[t] = sum_j y[pos(t, j)] + y[shared row t]
// (an expert shard skips pos = -1 and, without the shared expert, its row).
// The gate weights were already applied in the down-projection epilogue, so
// this is the sum of sglang-jax issue #1367 "Support Step 3.5 Flash",
// section "Model configuration" (MoE bullet: routed experts plus the shared
// expert).  Summed in fp32 in the fixed order j = 0..k-1 then the shared
// row, rounded once to the output dtype: deterministic.
#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {

namespace {

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

template <typename TO>
__global__ void __launch_bounds__(512) combine_kernel(const __nv_bfloat16* __restrict__ y,
                                                      const int* __restrict__ pos, int T, int k,
                                                      int H, int with_shared, TO* __restrict__ out) {
  pdl_wait();  // the previous kernel's results are visible
  __shared__ int rows[33];
  const int t = blockIdx.x;
  if (threadIdx.x < k) rows[threadIdx.x] = pos[static_cast<size_t>(t) * k + threadIdx.x];
  if (threadIdx.x == 0) rows[k] = with_shared ? T * k + t : -1;
  __syncthreads();
  const int nvec = H / 8;
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j <= k; ++j)  // (-1: another shard's expert, or no shared expert here)
      if (rows[j] >= 0) add8(acc, y + static_cast<size_t>(rows[j]) * H + v * 8);
    store8(out + static_cast<size_t>(t) * H + v * 8, acc);
  }
}

}  // namespace

cudaError_t launch_combine(const __nv_bfloat16* y, const int* pos, int T, int k, int H, bool out_bf16,
                           bool with_shared, void* out, cudaStream_t st) {
  const int threads = min(512, max(32, H / 8));
  if (out_bf16)
    return launch_pdl(combine_kernel<__nv_bfloat16>, dim3(T), dim3(threads), 0, st, y, pos, T, k, H,
                      with_shared ? 1 : 0, static_cast<__nv_bfloat16*>(out));
  return launch_pdl(combine_kernel<float>, dim3(T), dim3(threads), 0, st, y, pos, T, k, H,
                    with_shared ? 1 : 0, static_cast<float*>(out));
}

}  // namespace moe
