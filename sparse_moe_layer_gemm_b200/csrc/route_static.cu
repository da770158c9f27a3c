// moe_route_static: the routing stage (router logits, sigmoid scores, top-k on
// the biased scores, renormalised and scaled gate weights) for callers that
// must not allocate device memory.
//
// Who needs it: code that runs while a CUDA graph is being captured (a
// cudaMalloc there invalidates the capture), runtimes that own every byte of
// HBM through their own pool and forbid allocations behind their back, and
// latency-critical loops where a cudaMalloc / cudaFree may synchronise the
// whole device.  moe_forward needs a caller-provided workspace and a layer
// handle whose creation allocates; this entry point needs neither.
//
// Its only scratch, the split-K partial logits, lives in the file-scope array
// below.  A GPU holds it from the first call on that device (module loading
// may be lazy) until the process exits.  In host code `g_route_scratch` is a
// host-side stand-in, not a device address, so its device address is looked
// up with cudaGetSymbolAddress (with that device current) when a device is
// first seen, and again whenever the device's current CUDA context is not
// the one the address was taken in (after a cudaDeviceReset the module may
// be loaded at another address), then passed to the kernels.
#include <cudaTypedefs.h>
#include <math.h>

#include <mutex>

#include "../../include/moe.h"
#include "moe_internal.h"

namespace {

// 4 MiB: partial logits [splits][T][E] fp32.
constexpr size_t kRouteScratchFloats = static_cast<size_t>(1) << 20;
__device__ __align__(256) float g_route_scratch[kRouteScratchFloats];

constexpr int kMaxDevices = 64;
struct ScratchSlot {
  float* ptr;                 // device address of g_route_scratch
  unsigned long long ctx_id;  // the context it was taken in (0: unknown)
};
ScratchSlot g_scratch_dev[kMaxDevices] = {};
std::mutex g_scratch_mu;

// The unique id of the calling thread's current CUDA context (cuCtxGetId, a
// per-process counter that is never reused), through the driver entry points
// the runtime exposes; false if there is no current context or no entry point.
bool current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {  // (under g_scratch_mu)
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    looked_up = true;
  }
  if (get_current == nullptr || get_id == nullptr) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the scratch array on the current device: looked up the
// first time the device is seen and whenever its current context has changed
// since (or cannot be identified).
int scratch_for_current_device(float** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchSlot& slot = g_scratch_dev[dev];
  unsigned long long id = 0;
  const bool known = current_context_id(&id);
  if (slot.ptr == nullptr || !known || id != slot.ctx_id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr)
      return MOE_ERR_CUDA;
    // the lookup has made the device's primary context current if none was
    unsigned long long now = 0;
    slot.ptr = static_cast<float*>(p);
    slot.ctx_id = current_context_id(&now) ? now : 0;
  }
  *out = slot.ptr;
  return MOE_OK;
}

}  // namespace

extern "C" int moe_route_static(const void* x, int act_dtype, const float* router_w,
                                const float* router_bias, int T, int H, int E, int k,
                                int norm_expert_weight, float routed_scaling_factor,
                                int32_t* topk_idx, float* topk_w, void* stream) {
  if (T < 0 || H <= 0 || E <= 0 || k <= 0 || k > E) return MOE_ERR_INVALID_ARG;
  if (act_dtype != MOE_F32 && act_dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (!isfinite(routed_scaling_factor)) return MOE_ERR_INVALID_ARG;
  if (H % 128 != 0 || H > 16384 || E > 1024 || k > 32) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (x == nullptr || router_w == nullptr || topk_idx == nullptr || topk_w == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(x) % 16 != 0) return MOE_ERR_INVALID_ARG;
  // one split must fit: T * E fp32 partial logits
  if (static_cast<size_t>(T) * E > kRouteScratchFloats) return MOE_ERR_UNSUPPORTED;

  float* scratch = nullptr;
  int r = scratch_for_current_device(&scratch);
  if (r != MOE_OK) return r;
  // K splits: the rule moe_forward uses (fixed 128-wide K chunks), halved
  // until the partials fit the array; results equal moe_forward's whenever
  // no halving was needed (T * E * H / 128 <= 1,048,576).
  int splits = H / 128;
  while (splits > 1 && static_cast<size_t>(splits) * T * E > kRouteScratchFloats)
    splits = (splits % 2 == 0) ? splits / 2 : 1;

  // Every partial the top-k reads is written first, so nothing needs clearing.
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (moe::launch_router_logits(x, act_dtype == MOE_BF16, router_w, scratch, T, H, E, splits,
                                st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (moe::launch_topk(scratch, splits, T, E, k, router_bias, norm_expert_weight != 0,
                       routed_scaling_factor, topk_idx, topk_w, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
