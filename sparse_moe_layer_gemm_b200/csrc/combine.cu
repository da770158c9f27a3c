// K7: weighted combine.  out[t] = sum_j y[pos(t, j)] + y[shared row t]
// (an expert shard skips pos = -1 and, without the shared expert, its row).
// The gate weights were already applied in the down-projection epilogue, so
// this is the sum of sglang-jax issue #1367 "Support Step 3.5 Flash",
// section "Model configuration" (MoE bullet: routed experts plus the shared
// expert).  Summed in fp32 in the fixed order j = 0..k-1 then the shared
// row, rounded once to the output dtype: deterministic.  The rows y are bf16,
// or fp32 on the fp32 expert path.
#include "combine_device.cuh"
#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {

namespace {

// Every row of a token is loaded at once (combine_token): the bf16 -> bf16
// form fits two 512-thread blocks per SM in registers; the others take one.
template <typename TO, typename TY>
__global__ void __launch_bounds__(512, sizeof(TY) == 2 && sizeof(TO) == 2 ? 2 : 1)
    combine_kernel(const TY* __restrict__ y, const int* __restrict__ pos, int T, int k, int H,
                   int with_shared, TO* __restrict__ out) {
  pdl_wait();  // the previous kernel's results are visible
  __shared__ int rows[33];
  combine::combine_token<TO, TY>(blockIdx.x, y, pos, T, k, H, with_shared, out, rows);
}

template <typename TY>
cudaError_t launch_combine_t(const TY* y, const int* pos, int T, int k, int H, bool out_bf16,
                             bool with_shared, void* out, cudaStream_t st) {
  const int threads = min(512, max(32, H / 8));
  if (out_bf16)
    return launch_pdl(combine_kernel<__nv_bfloat16, TY>, dim3(T), dim3(threads), 0, st, y, pos,
                      T, k, H, with_shared ? 1 : 0, static_cast<__nv_bfloat16*>(out));
  return launch_pdl(combine_kernel<float, TY>, dim3(T), dim3(threads), 0, st, y, pos, T, k, H,
                    with_shared ? 1 : 0, static_cast<float*>(out));
}

}  // namespace

cudaError_t launch_combine(const __nv_bfloat16* y, const int* pos, int T, int k, int H, bool out_bf16,
                           bool with_shared, void* out, cudaStream_t st) {
  return launch_combine_t(y, pos, T, k, H, out_bf16, with_shared, out, st);
}

cudaError_t launch_combine_f32(const float* y, const int* pos, int T, int k, int H, bool out_bf16,
                               bool with_shared, void* out, cudaStream_t st) {
  return launch_combine_t(y, pos, T, k, H, out_bf16, with_shared, out, st);
}

}  // namespace moe
