// moe_check_wait_timeout: exercises the bounded-wait path every kernel relies
// on.  One CTA waits on an mbarrier that nothing arrives at, with a short
// limit; the wait must give up, set the timeout bit of a status word and let
// the kernel return, leaving the context usable.
#include "../../include/moe.h"
#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {
namespace {

__global__ void wait_timeout_kernel(uint64_t limit_ns, int* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
    // phase 0 never completes: no thread arrives
    if (mbar_wait(smem_u32(&bar), 0, nullptr, status, limit_ns)) atomicOr(status, 2);
  }
}

}  // namespace
}  // namespace moe

extern "C" int moe_check_wait_timeout(int limit_us, int* device_status) {
  if (limit_us <= 0 || limit_us > 10000000) return MOE_ERR_INVALID_ARG;
  int* status = nullptr;
  if (cudaMalloc(&status, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  int host = -1;
  bool ok = cudaMemset(status, 0, sizeof(int)) == cudaSuccess;
  if (ok) {
    moe::wait_timeout_kernel<<<1, 32>>>(static_cast<uint64_t>(limit_us) * 1000ull, status);
    ok = cudaGetLastError() == cudaSuccess && cudaDeviceSynchronize() == cudaSuccess &&
         cudaMemcpy(&host, status, sizeof(int), cudaMemcpyDeviceToHost) == cudaSuccess;
  }
  cudaFree(status);
  if (!ok) return MOE_ERR_CUDA;
  if (device_status != nullptr) *device_status = host;
  return host == moe::kDevErrTimeout ? MOE_OK : MOE_ERR_CUDA;
}
