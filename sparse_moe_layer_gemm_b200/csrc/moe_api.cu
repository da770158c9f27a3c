// C ABI of libmoe.so (declared in include/moe.h): argument checks, weight
// packing, workspace layout, tensor-map encoding and the stream-ordered
// launch sequence of the MoE FFN layer forward:
//   K1 router logits -> K2 top-k + weights -> K3 counting sort -> K4 gather
//   -> K5 grouped gate|up + SwiGLU -> K6 grouped down x gate weight -> K7 combine.
#include <cudaTypedefs.h>
#include <math.h>
#include <nvtx3/nvToolsExt.h>
#include <stdlib.h>
#include <string.h>

#include <new>
#include <vector>

#include "../../include/moe.h"
#include "api_util.h"
#include "moe_internal.h"

using moe::GemmParams;

struct moe_layer {
  moe_config_t cfg;
  int device;
  int num_sms;
  int I_pad;
  int fp8;              // expert weights are E4M3 codes (one byte each) + scales
  int f32;              // fp32 expert weights: the fp32 expert path (tf32 split)
  int first;            // expert shard: the layer holds experts [first, first + E_loc)
  int E_loc;            //   (E_loc = E: all of them)
  int with_shared;      //   and the shared expert if set
  void* w_gu;           // [(E+1) * 2 * I_pad, H] bf16 or E4M3 codes (fp32 path:
                        //   [.., 2H] fp32, the tf32 split's hi | lo halves)
  void* w_dn;           // [(E+1) * H, I_pad] bf16 or E4M3 codes (fp32 path: [.., 2 I_pad])
  float* sc_gu;         // FP8: scale of each packed gate|up row [(E+1) * 2 * I_pad]
  float* sc_dn;         // FP8: scale of each packed down row [(E+1) * H]
  float* router_w;      // [H, E]
  float* router_b;      // [E]
  __nv_bfloat16* router_tc;  // [E_pad, 3H]: bf16 three-term split of router_w^T
  float* router_t;           // [E, H]: router_w^T, fp32 (top-k candidate recomputation)
  int E_pad;
  int has_bias;
  int* status;          // device status word
  int loaded;
  CUtensorMap tm_gu;    // A operand of K5 (box 64 x 256)
  CUtensorMap tm_gu_pw;  // A operand of K5 on CTA pairs, wide stages (64 + 64 rows x 2 K blocks)
  CUtensorMap tm_gu_pn;  //   narrow stages (64 + 64 rows x 3 K blocks)
  CUtensorMap tm_dn;     // A operand of K6 (box 64 x 128)
  CUtensorMap tm_dn_pw;  // A operand of K6 on CTA pairs, wide stages (128 rows x 2 K blocks)
  CUtensorMap tm_dn_pn;  //   narrow stages (128 rows x 3 K blocks)
  CUtensorMap tm_router;  // A operand of the tensor-core router (box 64 x 128)
  CUtensorMap tm_rt_pw;   // the same for the fused kernel's pair MMAs: 128 rows x 2 K blocks
  CUtensorMap tm_rt_pn;   //   and x 3 K blocks
  int path;               // MOE_PATH_AUTO / MULTI / FUSED
  // stage timers: capacity x (MOE_NUM_STAGES + 1) events, filled in order
  std::vector<cudaEvent_t> events;
  int timing_capacity;
  int timing_recorded;
  // pipelined host forwards (moe_forward_host_async): input and output copy
  // streams, per staging slot the events "input copied", "forward done" and
  // "output copied", and the calls issued so far
  cudaStream_t st_in, st_out;
  cudaEvent_t ev_in[2], ev_fwd[2], ev_out[2];
  unsigned long long host_calls;
  int host_T;  // the last call's T (the staging slots' offsets depend on it)
};

namespace moe {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// bf16 [rows, cols] row-major, box = 64 columns (128 bytes) x box_rows, 128B
// swizzle; out-of-range elements read as zero.
bool encode_bf16_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(moe::kBK), box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_f32_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                   uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 4};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(moe::kBK32), box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bf16 [rows, cols] row-major seen as 3-D (64 columns, rows, cols / 64
// column blocks), box 64 x box_rows x kblocks column blocks, 128B swizzle:
// several K blocks of token rows (or weight rows) in one load (smem:
// k-block-major).
bool encode_bf16_kblocks(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                         uint32_t box_rows, uint32_t kblocks) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(moe::kBK), rows, cols / moe::kBK};
  cuuint64_t strides[2] = {cols * 2, static_cast<cuuint64_t>(moe::kBK) * 2};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(moe::kBK), box_rows, kblocks};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The packed gate|up weights as 4-D (64 columns, rows - 128, 2 halves 128
// rows apart, cols / 64 column blocks), box 64 x 64 x 2 x kblocks.
bool encode_bf16_gate_up_pair(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                              uint32_t kblocks) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr || rows < 2 * moe::kBM) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(moe::kBK), rows - moe::kBM, 2, cols / moe::kBK};
  cuuint64_t strides[3] = {cols * 2, static_cast<cuuint64_t>(moe::kBM) * cols * 2,
                           static_cast<cuuint64_t>(moe::kBK) * 2};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(moe::kBK), 64, 2, kblocks};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bf16 [rows, cols] row-major, box 32 columns x 16 rows, no swizzle: the
// expert GEMM epilogues' TMA stores of h and y.
bool encode_bf16_store(CUtensorMap* m, void* base, uint64_t rows, uint64_t cols) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {32, 16};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace moe

using moe::aligned;
using moe::DeviceGuard;
using moe::encode_bf16_2d;
using moe::encode_bf16_gate_up_pair;
using moe::encode_bf16_kblocks;
using moe::encode_bf16_kpair;
using moe::encode_bf16_store;
using moe::encode_f32_2d;

namespace {

// NVTX ranges of a forward's stages on the calling host thread (named in the
// timeline of a profiler; no cost without one).  At most one range is open;
// the destructor closes it on every return path.
struct NvtxStages {
  bool open = false;
  void enter(const char* name) {
    if (open) nvtxRangePop();
    nvtxRangePushA(name);
    open = true;
  }
  void leave() {
    if (open) nvtxRangePop();
    open = false;
  }
  ~NvtxStages() { leave(); }
};

const char* const kStageNames[MOE_NUM_STAGES] = {"moe router", "moe top-k", "moe sort",
                                                 "moe gather", "moe gate|up", "moe down",
                                                 "moe combine"};

constexpr int kMaxTokens = 1 << 20;
constexpr size_t kAlign = 1024;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct WsLayout {
  size_t partial, topk_idx, topk_w, masks, chunk_cnt, chunk_base, counts, row_start, tiles_gu,
      tiles_dn, perm, pos, w_perm, x_perm, h, y, local_idx, sync, total;
  int ksplit, nch, rows_routed, rows_xperm, rows_all;
};

// K splits of the CUDA-core router: fixed 128-wide K chunks, so a token's
// logits do not depend on the batch it arrives in; halved (or dropped to one)
// only if the partial logits would exceed 64 MB.
int router_ksplit(int T, int H, int E) {
  constexpr size_t kMaxPartialFloats = static_cast<size_t>(16) << 20;
  int s = H / 128;
  while (s > 1 && static_cast<size_t>(T) * E * s > kMaxPartialFloats) s = (s % 2 == 0) ? s / 2 : 1;
  return s;
}

WsLayout ws_layout(const moe_layer* L, int T) {
  const moe_config_t& c = L->cfg;
  const int H = c.hidden, E = c.num_experts, k = c.top_k, G = E + 1;
  WsLayout w{};
  w.ksplit = router_ksplit(T, H, E);
  w.nch = (T + moe::kSortChunk - 1) / moe::kSortChunk;
  w.rows_routed = T * k;
  // fp32 x, or the fp32 expert path: the shared expert's rows are in x_perm too
  w.rows_xperm = T * k + (c.act_dtype == MOE_F32 || L->f32 ? T : 0);
  w.rows_all = T * k + T;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, kAlign);
    return at;
  };
  // partial logits: the CUDA-core router's K splits, or the tensor-core
  // router's three parts
  const bool tc_router = c.act_dtype == MOE_BF16 && T >= moe::kTcRouterMinTokens;
  int parts = tc_router ? moe::kRouterTcParts : w.ksplit;
  // the fused path's router splits each bf16 term's K in two
  if (c.act_dtype == MOE_BF16 && T >= moe::kPairMinTokens && parts < moe::kFusedRouterParts)
    parts = moe::kFusedRouterParts;
  w.partial = take(static_cast<size_t>(parts) * T * E * sizeof(float));
  w.topk_idx = take(static_cast<size_t>(T) * k * sizeof(int));
  w.topk_w = take(static_cast<size_t>(T) * k * sizeof(float));
  w.masks = take(static_cast<size_t>(w.nch) * E * 4 * sizeof(uint32_t));
  w.chunk_cnt = take(static_cast<size_t>(w.nch) * E * sizeof(int));
  w.chunk_base = take(static_cast<size_t>(w.nch) * E * sizeof(int));
  w.counts = take(static_cast<size_t>(G) * sizeof(int));
  w.row_start = take(static_cast<size_t>(G + 1) * sizeof(int));
  w.tiles_gu = take(static_cast<size_t>(G + 1) * sizeof(int));
  w.tiles_dn = take(static_cast<size_t>(G + 1) * sizeof(int));
  w.perm = take(static_cast<size_t>(T) * k * sizeof(int));
  w.pos = take(static_cast<size_t>(T) * k * sizeof(int));
  w.w_perm = take(static_cast<size_t>(w.rows_all) * sizeof(float));
  // the fp32 expert path keeps x_perm and h as fp32 [hi | lo] and y as fp32
  const size_t xh = L->f32 ? 8 : 2, ye = L->f32 ? 4 : 2;
  w.x_perm = take(static_cast<size_t>(w.rows_xperm) * H * xh);
  w.h = take(static_cast<size_t>(w.rows_all) * L->I_pad * xh);
  w.y = take(static_cast<size_t>(w.rows_all) * H * ye);
  // expert shard: the selection in local expert ids (-1: another shard's)
  const bool shard = L->E_loc != E || L->first != 0;
  w.local_idx = shard ? take(static_cast<size_t>(T) * k * sizeof(int)) : 0;
  // fused path: the grid barrier's counter and the token blocks' readiness
  w.sync = take(moe::fused_sync_words(T, k, G) * sizeof(unsigned int));
  w.total = off;
  return w;
}

// The router part of both weight loaders (defined below).
int load_router(moe_layer* L, const float* router_w, const float* router_bias, cudaStream_t st);

// The fused forward gathers the routed rows into x_perm in a phase of its own
// (true) or lets its gather warps read them straight from x (false).  Measured
// on one B200 (prefill, T = 4096): 2.06 ms with the phase, 2.36 ms without.
constexpr bool kFusedGatherPhase = true;

// The fused persistent forward's conditions (see MOE_PATH_FUSED in moe.h).
bool fused_eligible(const moe_layer* L, int T) {
  const moe_config_t& c = L->cfg;
  return c.act_dtype == MOE_BF16 && !L->fp8 && !L->f32 && T >= moe::kPairMinTokens &&
         (c.hidden / moe::kBM) % 2 == 0 && c.num_experts <= moe::kFusedMaxExperts &&
         L->E_loc == c.num_experts && L->first == 0 && L->with_shared != 0;
}

// The optional routing outputs of a forward, copied from the workspace
// (a shard: counts and offsets of its own El experts).
int copy_routing(const moe_routing_t* routing, int T, int k, int El, const int* topk_idx,
                 const float* topk_w, const int* counts, const int* row_start, const int* perm,
                 cudaStream_t st) {
  if (routing == nullptr) return MOE_OK;
  const size_t tk = static_cast<size_t>(T) * k;
  if (routing->topk_idx)
    MOE_CUDA(cudaMemcpyAsync(routing->topk_idx, topk_idx, tk * 4, cudaMemcpyDeviceToDevice, st));
  if (routing->topk_w)
    MOE_CUDA(cudaMemcpyAsync(routing->topk_w, topk_w, tk * 4, cudaMemcpyDeviceToDevice, st));
  if (routing->counts)
    MOE_CUDA(cudaMemcpyAsync(routing->counts, counts, El * 4, cudaMemcpyDeviceToDevice, st));
  if (routing->offsets)
    MOE_CUDA(
        cudaMemcpyAsync(routing->offsets, row_start, (El + 1) * 4, cudaMemcpyDeviceToDevice, st));
  if (routing->perm)
    MOE_CUDA(cudaMemcpyAsync(routing->perm, perm, tk * 4, cudaMemcpyDeviceToDevice, st));
  return MOE_OK;
}

// The fused persistent forward (fused_moe.cu) on a checked workspace:
// zeroes the barrier and readiness counters, encodes the per-call tensor maps
// and launches the one kernel.  wait_ns / ready_extra: see FusedLaunch.
int launch_fused_forward(moe_layer* L, const void* x, int T, void* out, uint8_t* ws,
                         const WsLayout& w, cudaStream_t st, const moe_routing_t* routing,
                         uint64_t wait_ns, unsigned int ready_extra) {
  const moe_config_t& c = L->cfg;
  const int H = c.hidden, E = c.num_experts, k = c.top_k, Ip = L->I_pad, G = E + 1;
  float* partial = reinterpret_cast<float*>(ws + w.partial);
  int* topk_idx = reinterpret_cast<int*>(ws + w.topk_idx);
  float* topk_w = reinterpret_cast<float*>(ws + w.topk_w);
  uint32_t* masks = reinterpret_cast<uint32_t*>(ws + w.masks);
  int* chunk_cnt = reinterpret_cast<int*>(ws + w.chunk_cnt);
  int* chunk_base = reinterpret_cast<int*>(ws + w.chunk_base);
  int* counts = reinterpret_cast<int*>(ws + w.counts);
  int* row_start = reinterpret_cast<int*>(ws + w.row_start);
  int* tiles_gu = reinterpret_cast<int*>(ws + w.tiles_gu);
  int* tiles_dn = reinterpret_cast<int*>(ws + w.tiles_dn);
  int* perm = reinterpret_cast<int*>(ws + w.perm);
  int* pos = reinterpret_cast<int*>(ws + w.pos);
  float* w_perm = reinterpret_cast<float*>(ws + w.w_perm);
  __nv_bfloat16* hbuf = reinterpret_cast<__nv_bfloat16*>(ws + w.h);
  __nv_bfloat16* ybuf = reinterpret_cast<__nv_bfloat16*>(ws + w.y);
  moe::FusedLaunch f{};
  f.rt_w = L->tm_rt_pw;
  f.rt_n = L->tm_rt_pn;
  f.gu_w = L->tm_gu_pw;
  f.gu_n = L->tm_gu_pn;
  f.dn_w = L->tm_dn_pw;
  f.dn_n = L->tm_dn_pn;
  if (!encode_bf16_kblocks(&f.x_w, x, T, H, moe::kBN, 2) ||
      !encode_bf16_kblocks(&f.x_n, x, T, H, moe::kBBoxRows, 3) ||
      !encode_bf16_kblocks(&f.h_w, hbuf, w.rows_all, Ip, moe::kBN, 2) ||
      !encode_bf16_kblocks(&f.h_n, hbuf, w.rows_all, Ip, moe::kBBoxRows, 3) ||
      !encode_bf16_store(&f.st_h, hbuf, w.rows_all, Ip) ||
      !encode_bf16_store(&f.st_y, ybuf, w.rows_all, H))
    return MOE_ERR_CUDA;
  f.x = static_cast<const __nv_bfloat16*>(x);
  f.out = static_cast<__nv_bfloat16*>(out);
  f.T = T;
  f.H = H;
  f.E = E;
  f.k = k;
  f.I_pad = Ip;
  f.bias = L->has_bias ? L->router_b : nullptr;
  f.router_t = L->router_t;
  f.band = moe::router_refine_band(H);
  f.norm = c.norm_expert_weight != 0;
  f.scale = c.routed_scaling_factor;
  f.rt_mtiles = (L->E_pad + 2 * moe::kBM - 1) / (2 * moe::kBM);
  f.logits_out = routing != nullptr ? routing->logits : nullptr;
  f.partial = partial;
  f.topk_idx = topk_idx;
  f.topk_w = topk_w;
  f.masks = masks;
  f.chunk_cnt = chunk_cnt;
  f.chunk_base = chunk_base;
  f.counts = counts;
  f.row_start = row_start;
  f.tiles_gu = tiles_gu;
  f.tiles_dn = tiles_dn;
  f.perm = perm;
  f.pos = pos;
  f.w_perm = w_perm;
  f.h = hbuf;
  f.y = ybuf;
  f.sync = reinterpret_cast<unsigned int*>(ws + w.sync);
  f.limit = c.swiglu_limit;
  f.limit_shared = c.swiglu_limit_shared;
  f.status = L->status;
  f.wait_ns = wait_ns;
  f.ready_extra = ready_extra;
  if (kFusedGatherPhase) {
    f.x_perm = reinterpret_cast<__nv_bfloat16*>(ws + w.x_perm);
    if (!encode_bf16_kblocks(&f.xp_w, f.x_perm, w.rows_xperm, H, moe::kBN, 2) ||
        !encode_bf16_kblocks(&f.xp_n, f.x_perm, w.rows_xperm, H, moe::kBBoxRows, 3))
      return MOE_ERR_CUDA;
  }
  MOE_CUDA(cudaMemsetAsync(f.sync, 0, moe::fused_sync_words(T, k, G) * sizeof(unsigned int), st));
  MOE_CUDA(moe::launch_fused(f, st));
  return MOE_OK;
}

int forward_path(const moe_layer* L, int T) {
  if (L->path == MOE_PATH_FUSED && fused_eligible(L, T)) return MOE_PATH_FUSED;
  return MOE_PATH_MULTI;
}

}  // namespace

extern "C" {

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration or size";
    case MOE_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_DEVICE_TIMEOUT: return "a kernel gave up a bounded wait";
    case MOE_ERR_NOT_LOADED: return "weights not loaded";
    default: return "unknown status";
  }
}

int moe_config_check(const moe_config_t* c) {
  if (c == nullptr) return MOE_ERR_INVALID_ARG;
  if (c->hidden <= 0 || c->num_experts <= 0 || c->top_k <= 0 || c->intermediate <= 0 ||
      c->shared_intermediate <= 0)
    return MOE_ERR_INVALID_ARG;
  if ((c->act_dtype != MOE_F32 && c->act_dtype != MOE_BF16) ||
      (c->weight_dtype != MOE_F32 && c->weight_dtype != MOE_BF16 &&
       c->weight_dtype != MOE_FP8_E4M3))
    return MOE_ERR_INVALID_ARG;
  if (!isfinite(c->routed_scaling_factor) || !isfinite(c->swiglu_limit) ||
      !isfinite(c->swiglu_limit_shared) || c->swiglu_limit < 0.f || c->swiglu_limit_shared < 0.f)
    return MOE_ERR_INVALID_ARG;
  if (c->top_k > c->num_experts) return MOE_ERR_INVALID_ARG;
  if (c->hidden % 128 != 0 || c->hidden > 16384) return MOE_ERR_UNSUPPORTED;
  if (c->num_experts > moe::kMaxGroups - 1 || c->top_k > 32 || c->intermediate > 8192) return MOE_ERR_UNSUPPORTED;
  if (c->shared_intermediate != c->intermediate) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

int moe_create(const moe_config_t* cfg, moe_layer_t** out) {
  if (cfg == nullptr) {
    if (out != nullptr) *out = nullptr;
    return MOE_ERR_INVALID_ARG;
  }
  return moe_create_shard(cfg, 0, cfg->num_experts, 1, out);
}

int moe_create_shard(const moe_config_t* cfg, int expert_first, int expert_count,
                     int with_shared, moe_layer_t** out) {
  if (out == nullptr) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  const int chk = moe_config_check(cfg);
  if (chk != MOE_OK) return chk;
  if (expert_first < 0 || expert_count < 1 || expert_first + expert_count > cfg->num_experts ||
      (with_shared != 0 && with_shared != 1))
    return MOE_ERR_INVALID_ARG;
  moe_layer* L = new (std::nothrow) moe_layer();
  if (L == nullptr) return MOE_ERR_CUDA;
  L->cfg = *cfg;
  L->first = expert_first;
  L->E_loc = expert_count;
  L->with_shared = with_shared;
  L->fp8 = cfg->weight_dtype == MOE_FP8_E4M3 ? 1 : 0;
  L->f32 = cfg->weight_dtype == MOE_F32 ? 1 : 0;
  L->I_pad = (cfg->intermediate + 127) / 128 * 128;
  L->E_pad = (cfg->num_experts + 127) / 128 * 128;
  if (cudaGetDevice(&L->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&L->num_sms, cudaDevAttrMultiProcessorCount, L->device) !=
          cudaSuccess) {
    delete L;
    return MOE_ERR_CUDA;
  }
  // expert weights: the shard's experts + the shared expert (group E_loc);
  // the router covers all experts
  const size_t H = cfg->hidden, E = cfg->num_experts, Ip = L->I_pad, El = L->E_loc;
  const size_t el = L->fp8 ? 1 : L->f32 ? 8 : 2;  // bytes per weight (fp32: hi + lo)
  const size_t gu_bytes = (El + 1) * 2 * Ip * H * el, dn_bytes = (El + 1) * H * Ip * el;
  if (moe::gemm_configure_device() != cudaSuccess ||
      moe::gemm_fp8_configure_device() != cudaSuccess ||
      moe::gemm_pair_configure_device(L->num_sms) != cudaSuccess ||
      moe::fused_configure_device(L->num_sms) != cudaSuccess ||
      moe::topk_configure_device() != cudaSuccess ||
      moe::gather_configure_device() != cudaSuccess ||
      cudaMalloc(&L->w_gu, gu_bytes) != cudaSuccess ||
      cudaMalloc(&L->w_dn, dn_bytes) != cudaSuccess ||
      cudaMalloc(&L->router_w, H * E * sizeof(float)) != cudaSuccess ||
      cudaMalloc(&L->router_b, E * sizeof(float)) != cudaSuccess ||
      cudaMalloc(&L->router_tc, static_cast<size_t>(L->E_pad) * 3 * H * 2) != cudaSuccess ||
      cudaMalloc(&L->router_t, E * H * sizeof(float)) != cudaSuccess ||
      cudaMalloc(&L->status, sizeof(int)) != cudaSuccess ||
      cudaMemset(L->status, 0, sizeof(int)) != cudaSuccess ||
      (L->fp8 && (cudaMalloc(&L->sc_gu, (El + 1) * 2 * Ip * sizeof(float)) != cudaSuccess ||
                  cudaMalloc(&L->sc_dn, (El + 1) * H * sizeof(float)) != cudaSuccess))) {
    moe_destroy(L);
    return MOE_ERR_CUDA;
  }
  // (FP8 codes are read with plain bulk copies: no tensor maps)
  const bool maps_ok =
      L->fp8 ||
      (L->f32 && encode_f32_2d(&L->tm_gu, L->w_gu, (El + 1) * 2 * Ip, 2 * H, 2 * moe::kBM) &&
       encode_f32_2d(&L->tm_dn, L->w_dn, (El + 1) * H, 2 * Ip, moe::kBM)) ||
      (!L->f32 && encode_bf16_2d(&L->tm_gu, L->w_gu, (El + 1) * 2 * Ip, H, 2 * moe::kBM) &&
       encode_bf16_gate_up_pair(&L->tm_gu_pw, L->w_gu, (El + 1) * 2 * Ip, H, 2) &&
       encode_bf16_gate_up_pair(&L->tm_gu_pn, L->w_gu, (El + 1) * 2 * Ip, H, 3) &&
       encode_bf16_2d(&L->tm_dn, L->w_dn, (El + 1) * H, Ip, moe::kBM) &&
       encode_bf16_kblocks(&L->tm_dn_pw, L->w_dn, (El + 1) * H, Ip, moe::kBM, 2) &&
       encode_bf16_kblocks(&L->tm_dn_pn, L->w_dn, (El + 1) * H, Ip, moe::kBM, 3));
  if (!maps_ok || !encode_bf16_2d(&L->tm_router, L->router_tc, L->E_pad, 3 * H, moe::kBM) ||
      !encode_bf16_kblocks(&L->tm_rt_pw, L->router_tc, L->E_pad, 3 * H, moe::kBM, 2) ||
      !encode_bf16_kblocks(&L->tm_rt_pn, L->router_tc, L->E_pad, 3 * H, moe::kBM, 3)) {
    moe_destroy(L);
    return MOE_ERR_CUDA;
  }
  *out = L;
  return MOE_OK;
}

}  // extern "C"

namespace {

// Packs the bf16 / fp32 expert weights: the layer's E_loc routed experts start
// first_in_tensor experts into the caller's tensors (the shard's own first
// expert for moe_load_weights, 0 for moe_load_shard_weights), then the shared
// expert if the layer holds it, then the router.  fp32 weights become the
// fp32 expert path's [hi | lo] rows.
int load_bf16(moe_layer* L, const float* router_w, const float* router_bias, const void* w_gate,
              const void* w_up, const void* w_down, const void* sh_gate, const void* sh_up,
              const void* sh_down, size_t first_in_tensor, cudaStream_t st) {
  const moe_config_t& c = L->cfg;
  const int H = c.hidden, El = L->E_loc, I = c.intermediate, Ip = L->I_pad;
  const bool wb = c.weight_dtype == MOE_BF16;
  const size_t gu_group = static_cast<size_t>(2) * Ip * H, dn_group = static_cast<size_t>(H) * Ip;
  if (L->f32) {
    // two fp32 values per weight: groups of 2 * gu_group / 2 * dn_group floats
    const size_t off = first_in_tensor * H * I * 4;
    const uint8_t* wg = static_cast<const uint8_t*>(w_gate) + off;
    const uint8_t* wu = static_cast<const uint8_t*>(w_up) + off;
    const uint8_t* wd = static_cast<const uint8_t*>(w_down) + off;
    float* gu = static_cast<float*>(L->w_gu);
    float* dn = static_cast<float*>(L->w_dn);
    MOE_CUDA(cudaMemsetAsync(gu, 0, (El + 1) * gu_group * 8, st));
    MOE_CUDA(cudaMemsetAsync(dn, 0, (El + 1) * dn_group * 8, st));
    MOE_CUDA(moe::launch_pack_gate_up_split(wg, false, El, H, I, Ip, 0, gu, st));
    MOE_CUDA(moe::launch_pack_gate_up_split(wu, false, El, H, I, Ip, 1, gu, st));
    MOE_CUDA(moe::launch_pack_down_split(wd, false, El, H, I, Ip, dn, st));
    if (L->with_shared) {
      float* gsh = gu + El * 2 * gu_group;
      MOE_CUDA(moe::launch_pack_gate_up_split(sh_gate, false, 1, H, I, Ip, 0, gsh, st));
      MOE_CUDA(moe::launch_pack_gate_up_split(sh_up, false, 1, H, I, Ip, 1, gsh, st));
      MOE_CUDA(moe::launch_pack_down_split(sh_down, false, 1, H, I, Ip, dn + El * 2 * dn_group,
                                           st));
    }
    return load_router(L, router_w, router_bias, st);
  }
  __nv_bfloat16* gu = static_cast<__nv_bfloat16*>(L->w_gu);
  __nv_bfloat16* dn = static_cast<__nv_bfloat16*>(L->w_dn);
  const size_t off = first_in_tensor * H * I * (wb ? 2 : 4);
  const uint8_t* wg = static_cast<const uint8_t*>(w_gate) + off;
  const uint8_t* wu = static_cast<const uint8_t*>(w_up) + off;
  const uint8_t* wd = static_cast<const uint8_t*>(w_down) + off;
  MOE_CUDA(cudaMemsetAsync(gu, 0, (El + 1) * gu_group * 2, st));
  MOE_CUDA(cudaMemsetAsync(dn, 0, (El + 1) * dn_group * 2, st));
  MOE_CUDA(moe::launch_pack_gate_up(wg, wb, El, H, I, Ip, 0, gu, st));
  MOE_CUDA(moe::launch_pack_gate_up(wu, wb, El, H, I, Ip, 1, gu, st));
  MOE_CUDA(moe::launch_pack_down(wd, wb, El, H, I, Ip, dn, st));
  if (L->with_shared) {
    MOE_CUDA(moe::launch_pack_gate_up(sh_gate, wb, 1, H, I, Ip, 0, gu + El * gu_group, st));
    MOE_CUDA(moe::launch_pack_gate_up(sh_up, wb, 1, H, I, Ip, 1, gu + El * gu_group, st));
    MOE_CUDA(moe::launch_pack_down(sh_down, wb, 1, H, I, Ip, dn + El * dn_group, st));
  }
  return load_router(L, router_w, router_bias, st);
}

}  // namespace

extern "C" {

int moe_load_weights(moe_layer_t* L, const float* router_w, const float* router_bias,
                     const void* w_gate, const void* w_up, const void* w_down, const void* sh_gate,
                     const void* sh_up, const void* sh_down, void* stream) {
  if (L == nullptr || router_w == nullptr || w_gate == nullptr || w_up == nullptr ||
      w_down == nullptr || sh_gate == nullptr || sh_up == nullptr || sh_down == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (L->fp8) return MOE_ERR_INVALID_ARG;  // codes need their scales: moe_load_weights_fp8
  DeviceGuard dg(L->device);
  if (!dg.ok) return MOE_ERR_CUDA;
  // the shard's experts start `first` experts into the caller's tensors
  return load_bf16(L, router_w, router_bias, w_gate, w_up, w_down, sh_gate, sh_up, sh_down,
                   static_cast<size_t>(L->first), static_cast<cudaStream_t>(stream));
}

int moe_load_shard_weights(moe_layer_t* L, const float* router_w, const float* router_bias,
                           const void* w_gate, const void* w_up, const void* w_down,
                           const void* sh_gate, const void* sh_up, const void* sh_down,
                           void* stream) {
  if (L == nullptr || router_w == nullptr || w_gate == nullptr || w_up == nullptr ||
      w_down == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (L->with_shared && (sh_gate == nullptr || sh_up == nullptr || sh_down == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (L->fp8) return MOE_ERR_INVALID_ARG;
  DeviceGuard dg(L->device);
  if (!dg.ok) return MOE_ERR_CUDA;
  return load_bf16(L, router_w, router_bias, w_gate, w_up, w_down, sh_gate, sh_up, sh_down, 0,
                   static_cast<cudaStream_t>(stream));
}

int moe_load_weights_fp8(moe_layer_t* L, const float* router_w, const float* router_bias,
                         const uint8_t* w_gate, const uint8_t* w_up, const uint8_t* w_down,
                         const float* s_gate, const float* s_up, const float* s_down,
                         const uint8_t* sh_gate, const uint8_t* sh_up, const uint8_t* sh_down,
                         const float* sh_s_gate, const float* sh_s_up, const float* sh_s_down,
                         void* stream) {
  if (L == nullptr || router_w == nullptr || w_gate == nullptr || w_up == nullptr ||
      w_down == nullptr || s_gate == nullptr || s_up == nullptr || s_down == nullptr ||
      sh_gate == nullptr || sh_up == nullptr || sh_down == nullptr || sh_s_gate == nullptr ||
      sh_s_up == nullptr || sh_s_down == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (!L->fp8) return MOE_ERR_INVALID_ARG;
  DeviceGuard dg(L->device);
  if (!dg.ok) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const moe_config_t& c = L->cfg;
  const int H = c.hidden, El = L->E_loc, I = c.intermediate, Ip = L->I_pad;
  const size_t gu_group = static_cast<size_t>(2) * Ip * H, dn_group = static_cast<size_t>(H) * Ip;
  uint8_t* gu = static_cast<uint8_t*>(L->w_gu);
  uint8_t* dn = static_cast<uint8_t*>(L->w_dn);
  // the shard's experts start `first` experts into the caller's tensors
  const size_t f = static_cast<size_t>(L->first);
  const size_t off = f * H * I;
  // padded rows and columns: code 0 (value 0), scale 0
  MOE_CUDA(cudaMemsetAsync(gu, 0, (El + 1) * gu_group, st));
  MOE_CUDA(cudaMemsetAsync(dn, 0, (El + 1) * dn_group, st));
  MOE_CUDA(cudaMemsetAsync(L->sc_gu, 0, (El + 1) * 2 * Ip * sizeof(float), st));
  MOE_CUDA(cudaMemsetAsync(L->sc_dn, 0, (El + 1) * H * sizeof(float), st));
  MOE_CUDA(moe::launch_pack_codes_gate_up(w_gate + off, El, H, I, Ip, 0, gu, st));
  MOE_CUDA(moe::launch_pack_codes_gate_up(w_up + off, El, H, I, Ip, 1, gu, st));
  const int dn_rows = moe::kBM * moe::gemm_down_blocks(H);  // the down GEMM's tile rows
  MOE_CUDA(moe::launch_pack_codes_down(w_down + off, El, H, I, Ip, dn_rows, dn, st));
  MOE_CUDA(moe::launch_pack_gate_up_scales(s_gate + f * I, El, I, Ip, 0, L->sc_gu, st));
  MOE_CUDA(moe::launch_pack_gate_up_scales(s_up + f * I, El, I, Ip, 1, L->sc_gu, st));
  MOE_CUDA(cudaMemcpyAsync(L->sc_dn, s_down + f * H, static_cast<size_t>(El) * H * sizeof(float),
                           cudaMemcpyDeviceToDevice, st));
  if (L->with_shared) {
    float* sgu_sh = L->sc_gu + static_cast<size_t>(El) * 2 * Ip;
    MOE_CUDA(moe::launch_pack_codes_gate_up(sh_gate, 1, H, I, Ip, 0, gu + El * gu_group, st));
    MOE_CUDA(moe::launch_pack_codes_gate_up(sh_up, 1, H, I, Ip, 1, gu + El * gu_group, st));
    MOE_CUDA(moe::launch_pack_codes_down(sh_down, 1, H, I, Ip, dn_rows, dn + El * dn_group, st));
    MOE_CUDA(moe::launch_pack_gate_up_scales(sh_s_gate, 1, I, Ip, 0, sgu_sh, st));
    MOE_CUDA(moe::launch_pack_gate_up_scales(sh_s_up, 1, I, Ip, 1, sgu_sh, st));
    MOE_CUDA(cudaMemcpyAsync(L->sc_dn + static_cast<size_t>(El) * H, sh_s_down,
                             H * sizeof(float), cudaMemcpyDeviceToDevice, st));
  }
  return load_router(L, router_w, router_bias, st);
}

int moe_decode_e4m3(const uint8_t* codes, size_t n, uint16_t* out, void* stream) {
  if (n == 0) return MOE_OK;
  if (codes == nullptr || out == nullptr || n % 4 != 0 || !aligned(codes, 16) || !aligned(out, 16))
    return MOE_ERR_INVALID_ARG;
  MOE_CUDA(moe::launch_decode_e4m3(codes, n, reinterpret_cast<__nv_bfloat16*>(out),
                                   static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

}  // extern "C"

namespace {

// The router weight and bias: kept fp32, plus the tensor-core router's bf16
// three-term split and the fp32 transpose.
int load_router(moe_layer* L, const float* router_w, const float* router_bias, cudaStream_t st) {
  const moe_config_t& c = L->cfg;
  const int H = c.hidden, E = c.num_experts;
  MOE_CUDA(cudaMemcpyAsync(L->router_w, router_w, static_cast<size_t>(H) * E * sizeof(float),
                           cudaMemcpyDeviceToDevice, st));
  MOE_CUDA(moe::launch_pack_router(router_w, H, E, L->E_pad, L->router_tc, L->router_t, st));
  L->has_bias = (c.use_router_bias && router_bias != nullptr) ? 1 : 0;
  if (L->has_bias)
    MOE_CUDA(cudaMemcpyAsync(L->router_b, router_bias, E * sizeof(float),
                             cudaMemcpyDeviceToDevice, st));
  L->loaded = 1;
  return MOE_OK;
}

}  // namespace

extern "C" {

int moe_workspace_size(const moe_layer_t* L, int T, size_t* bytes) {
  if (L == nullptr || bytes == nullptr || T < 0) return MOE_ERR_INVALID_ARG;
  if (T > kMaxTokens) return MOE_ERR_UNSUPPORTED;
  *bytes = (T == 0) ? 0 : ws_layout(L, T).total;
  return MOE_OK;
}

int moe_workspace_size_host(const moe_layer_t* L, int T, size_t* bytes) {
  size_t b = 0;
  const int r = moe_workspace_size(L, T, &b);
  if (r != MOE_OK) return r;
  const size_t el = (L->cfg.act_dtype == MOE_BF16) ? 2 : 4;
  const size_t io = align_up(static_cast<size_t>(T) * L->cfg.hidden * el, kAlign);
  *bytes = b + 4 * io;  // two staging slots of (x, out)
  return MOE_OK;
}

int moe_forward(moe_layer_t* L, const void* x, int T, void* out, void* workspace, size_t ws_bytes,
                void* stream, const moe_routing_t* routing) {
  if (L == nullptr || T < 0) return MOE_ERR_INVALID_ARG;
  if (T > kMaxTokens) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (x == nullptr || out == nullptr || x == out) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(out, 16)) return MOE_ERR_INVALID_ARG;
  if (!L->loaded) return MOE_ERR_NOT_LOADED;
  const WsLayout w = ws_layout(L, T);
  if (workspace == nullptr || ws_bytes < w.total || !aligned(workspace, 256))
    return MOE_ERR_WORKSPACE;
  DeviceGuard dg(L->device);
  if (!dg.ok) return MOE_ERR_CUDA;

  const moe_config_t& c = L->cfg;
  // E: all experts (router, selection); El: this layer's experts (a shard
  // holds [first, first + El)); G: its groups (the shared expert is group El)
  const int H = c.hidden, E = c.num_experts, k = c.top_k, Ip = L->I_pad;
  const int El = L->E_loc, G = El + 1;
  const bool shard = El != E || L->first != 0;
  const bool xb = c.act_dtype == MOE_BF16;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* partial = reinterpret_cast<float*>(ws + w.partial);
  int* topk_idx = reinterpret_cast<int*>(ws + w.topk_idx);
  float* topk_w = reinterpret_cast<float*>(ws + w.topk_w);
  uint32_t* masks = reinterpret_cast<uint32_t*>(ws + w.masks);
  int* chunk_cnt = reinterpret_cast<int*>(ws + w.chunk_cnt);
  int* chunk_base = reinterpret_cast<int*>(ws + w.chunk_base);
  int* counts = reinterpret_cast<int*>(ws + w.counts);
  int* row_start = reinterpret_cast<int*>(ws + w.row_start);
  int* tiles_gu = reinterpret_cast<int*>(ws + w.tiles_gu);
  int* tiles_dn = reinterpret_cast<int*>(ws + w.tiles_dn);
  int* perm = reinterpret_cast<int*>(ws + w.perm);
  int* pos = reinterpret_cast<int*>(ws + w.pos);
  float* w_perm = reinterpret_cast<float*>(ws + w.w_perm);
  __nv_bfloat16* x_perm = reinterpret_cast<__nv_bfloat16*>(ws + w.x_perm);
  __nv_bfloat16* hbuf = reinterpret_cast<__nv_bfloat16*>(ws + w.h);
  __nv_bfloat16* ybuf = reinterpret_cast<__nv_bfloat16*>(ws + w.y);

  cudaEvent_t* ev = nullptr;
  if (L->timing_capacity > 0 && L->timing_recorded < L->timing_capacity)
    ev = &L->events[static_cast<size_t>(L->timing_recorded++) * (MOE_NUM_STAGES + 1)];
  NvtxStages nvtx;
  auto mark = [&](int i) {
    if (i < MOE_NUM_STAGES)
      nvtx.enter(kStageNames[i]);
    else
      nvtx.leave();
    return ev == nullptr ? cudaSuccess : cudaEventRecord(ev[i], st);
  };

  if (forward_path(L, T) == MOE_PATH_FUSED) {
    // one persistent kernel (fused_moe.cu); the whole forward is stage 0
    MOE_CUDA(mark(0));
    nvtx.enter("moe fused forward");
    const int r = launch_fused_forward(L, x, T, out, ws, w, st, routing, 0, 0);
    if (r != MOE_OK) return r;
    for (int i = 1; i <= MOE_NUM_STAGES; ++i) MOE_CUDA(mark(i));
    return copy_routing(routing, T, k, El, topk_idx, topk_w, counts, row_start, perm, st);
  }

  // expert-GEMM tiles: on one SM, 128 tokens x gate|up one 128-feature block
  // (down one or two); on CTA pairs (large T), 256 tokens x gate|up 128
  // features (down 256)
  // (FP8 weights: always the one-SM tiles, which expand the codes; so does
  // the fp32 expert path, on tf32)
  const bool f32 = L->f32 != 0;
  const bool pair_gu = !L->fp8 && !f32 && T >= moe::kPairMinTokens;
  const bool pair_dn = !L->fp8 && !f32 && T >= moe::kPairMinTokens && (H / moe::kBM) % 2 == 0;
  const int dn_blocks = moe::gemm_down_blocks(H);
  const int bn_gu = L->fp8 ? moe::kFp8BN : pair_gu ? 2 * moe::kBN : moe::kBN;
  const int bn_dn = L->fp8 ? moe::kFp8BN : pair_dn ? 2 * moe::kBN : moe::kBN;
  const int mt_gu = Ip / moe::kBM;
  const int mt_dn = pair_dn ? H / (2 * moe::kBM) : H / moe::kBM / dn_blocks;

  // Token-row operands, each with kBBoxRows- and kBN-row boxes: x_perm (or x
  // for the shared expert) for K5 and the router, h for K6.  The CTA-pair
  // kernels read them as K-block maps (32 rows x 3 K blocks, 128 rows x 2).
  moe::GemmMaps gu{}, dn{}, rt{};
  const bool maps_ok = [&] {
    if (f32) {
      // fp32 expert path: [hi | lo] rows of x_perm (the shared rows included)
      // and of h; the router keeps its own path below
      gu.a = L->tm_gu;
      dn.a = L->tm_dn;
      if (!encode_f32_2d(&gu.b, x_perm, w.rows_xperm, 2 * H, moe::kBBoxRows) ||
          !encode_f32_2d(&gu.bw, x_perm, w.rows_xperm, 2 * H, moe::kBN) ||
          !encode_f32_2d(&dn.b, hbuf, w.rows_all, 2 * Ip, moe::kBBoxRows) ||
          !encode_f32_2d(&dn.bw, hbuf, w.rows_all, 2 * Ip, moe::kBN))
        return false;
      gu.bsh = gu.b;
      gu.bshw = gu.bw;
      dn.bsh = dn.b;
      dn.bshw = dn.bw;
      gu.out = gu.b;  // not read
      dn.out = dn.b;
      rt.a = L->tm_router;
      rt.out = dn.b;
      if (xb && (!encode_bf16_2d(&rt.b, x, T, H, moe::kBBoxRows) ||
                 !encode_bf16_2d(&rt.bw, x, T, H, moe::kBN)))
        return false;
      return true;
    }
    if (pair_gu) {
      gu.a = L->tm_gu_pw;
      gu.a2 = L->tm_gu_pn;
      if (!encode_bf16_kblocks(&gu.b, x_perm, w.rows_xperm, H, moe::kBBoxRows, 3) ||
          !encode_bf16_kblocks(&gu.bw, x_perm, w.rows_xperm, H, moe::kBN, 2))
        return false;
      if (xb) {
        if (!encode_bf16_kblocks(&gu.bsh, x, T, H, moe::kBBoxRows, 3) ||
            !encode_bf16_kblocks(&gu.bshw, x, T, H, moe::kBN, 2))
          return false;
      } else {
        gu.bsh = gu.b;
        gu.bshw = gu.bw;
      }
    } else {
      gu.a = L->tm_gu;  // (unused with FP8 weights)
      if (!encode_bf16_2d(&gu.b, x_perm, w.rows_xperm, H, moe::kBBoxRows) ||
          !encode_bf16_2d(&gu.bw, x_perm, w.rows_xperm, H, moe::kBN))
        return false;
      if (xb) {
        if (!encode_bf16_2d(&gu.bsh, x, T, H, moe::kBBoxRows) ||
            !encode_bf16_2d(&gu.bshw, x, T, H, moe::kBN))
          return false;
      } else {
        gu.bsh = gu.b;
        gu.bshw = gu.bw;
      }
    }
    if (pair_dn) {
      dn.a = L->tm_dn_pw;
      dn.a2 = L->tm_dn_pn;
      if (!encode_bf16_kblocks(&dn.b, hbuf, w.rows_all, Ip, moe::kBBoxRows, 3) ||
          !encode_bf16_kblocks(&dn.bw, hbuf, w.rows_all, Ip, moe::kBN, 2))
        return false;
    } else {
      dn.a = L->tm_dn;
      if (!encode_bf16_2d(&dn.b, hbuf, w.rows_all, Ip, moe::kBBoxRows) ||
          !encode_bf16_2d(&dn.bw, hbuf, w.rows_all, Ip, moe::kBN))
        return false;
    }
    dn.bsh = dn.b;
    dn.bshw = dn.bw;
    if (!encode_bf16_store(&gu.out, hbuf, w.rows_all, Ip) ||
        !encode_bf16_store(&dn.out, ybuf, w.rows_all, H))
      return false;
    // the tensor-core router (bf16 x): the one-SM kernel's 2-D maps of x
    rt.a = L->tm_router;
    rt.out = dn.out;  // unused by the router
    if (xb && (!encode_bf16_2d(&rt.b, x, T, H, moe::kBBoxRows) ||
               !encode_bf16_2d(&rt.bw, x, T, H, moe::kBN)))
      return false;
    return true;
  }();
  if (!maps_ok) return MOE_ERR_CUDA;
  moe::GemmMaps gu8{}, dn8{};  // FP8 GEMMs: token rows as k-pair maps
  if (L->fp8) {
    gu8.out = gu.out;
    dn8.out = dn.out;
    if (!encode_bf16_kpair(&gu8.b, x_perm, w.rows_xperm, H, moe::kFp8BN) ||
        !encode_bf16_kpair(&dn8.b, hbuf, w.rows_all, Ip, moe::kFp8BN) ||
        (xb && !encode_bf16_kpair(&gu8.bsh, x, T, H, moe::kFp8BN)))
      return MOE_ERR_CUDA;
    if (!xb) gu8.bsh = gu8.b;
    dn8.bsh = dn8.b;
  }

  MOE_CUDA(mark(0));
  int ksplit = w.ksplit;
  moe::TopkRefine refine{};
  const bool tc_router = xb && T >= moe::kTcRouterMinTokens;
  if (tc_router) {
    // tensor-core router: one group of T rows; the K = 3H reduction over
    // W1 | W2 | W3 runs as three parts (three times the tiles, a third of the
    // k-blocks each), summed in fixed order by the top-k
    GemmParams r{};
    r.single_rows = T;
    r.E = E;
    r.num_kb = H / moe::kBK;
    r.m_tiles = L->E_pad / moe::kBM;
    r.k_parts = moe::kRouterTcParts;
    r.part_stride = static_cast<size_t>(T) * E;
    r.out_f32 = partial;
    r.out_ld = E;
    r.valid_feats = E;
    r.out_feats = E;
    r.status = L->status;
    const int tiles = r.k_parts * r.m_tiles * ((T + 2 * moe::kBN - 1) / (2 * moe::kBN));  // 256-token tiles
    MOE_CUDA(moe::launch_gemm_router(rt, r, tiles < L->num_sms ? tiles : L->num_sms, st));
    ksplit = moe::kRouterTcParts;
    refine.x = static_cast<const __nv_bfloat16*>(x);
    refine.w_t = L->router_t;
    refine.H = H;
    refine.band = moe::router_refine_band(H);
  } else {
    MOE_CUDA(moe::launch_router_logits(x, xb, L->router_w, partial, T, H, E, w.ksplit, st));
  }
  MOE_CUDA(mark(1));
  MOE_CUDA(moe::launch_topk(partial, ksplit, T, E, k, L->has_bias ? L->router_b : nullptr,
                            c.norm_expert_weight != 0, c.routed_scaling_factor, topk_idx, topk_w,
                            st, routing != nullptr ? routing->logits : nullptr,
                            tc_router ? &refine : nullptr));
  MOE_CUDA(mark(2));
  const int* sel = topk_idx;  // the selection in this layer's expert ids
  if (shard) {
    int* local_idx = reinterpret_cast<int*>(ws + w.local_idx);
    MOE_CUDA(moe::launch_localize(topk_idx, T * k, L->first, El, local_idx, st));
    sel = local_idx;
  }
  MOE_CUDA(moe::launch_sort(sel, topk_w, T, k, El, L->with_shared ? T : 0, bn_gu, bn_dn, mt_gu,
                            mt_dn, masks, chunk_cnt, chunk_base, counts, row_start, tiles_gu,
                            tiles_dn, perm, pos, w_perm, st));
  MOE_CUDA(mark(3));
  if (f32)
    MOE_CUDA(moe::launch_gather_split(x, xb, perm, w.rows_routed, k, T, H,
                                      reinterpret_cast<float*>(ws + w.x_perm), L->num_sms, st));
  else
    MOE_CUDA(moe::launch_gather(x, xb, perm, pos, w.rows_routed, k, T, H, !xb, x_perm,
                                L->num_sms, L->status, st));
  MOE_CUDA(mark(4));

  GemmParams p{};
  p.counts = counts;
  p.row_start = row_start;
  p.G = G;
  p.E = El;
  p.status = L->status;
  p.limit = c.swiglu_limit;
  p.limit_shared = c.swiglu_limit_shared;

  p.tile_start = tiles_gu;
  p.num_kb = H / moe::kBK;
  p.m_tiles = mt_gu;
  p.a_rows_per_group = 2 * Ip;
  p.shared_b_row0 = xb ? 0 : T * k;
  p.out = hbuf;
  p.out_ld = Ip;
  p.out_feats = Ip;
  p.w_perm = nullptr;
  p.a_scale = L->fp8 ? L->sc_gu : nullptr;
  p.a_codes = L->fp8 ? static_cast<const uint8_t*>(L->w_gu) : nullptr;
  if (f32) {
    // three terms of H / 32 k-blocks; h as fp32 [hi | lo] rows of 2 I_pad
    p.kb_term = H / moe::kBK32;
    p.num_kb = 3 * p.kb_term;
    p.shared_b_row0 = T * k;
    p.out = nullptr;
    p.out_f32 = reinterpret_cast<float*>(ws + w.h);
    p.out_ld = 2 * Ip;
  }
  MOE_CUDA(f32       ? moe::launch_gemm_gate_up_tf32(gu, p, L->num_sms, st)
           : L->fp8  ? moe::launch_gemm_gate_up_fp8(gu8, p, L->num_sms, st)
           : pair_gu ? moe::launch_gemm_gate_up_pair(gu, p, st)
                     : moe::launch_gemm_gate_up(gu, p, L->num_sms, st));
  MOE_CUDA(mark(5));

  p.tile_start = tiles_dn;
  p.num_kb = Ip / moe::kBK;
  p.m_tiles = mt_dn;
  p.a_rows_per_group = H;
  p.shared_b_row0 = T * k;
  p.out = ybuf;
  p.out_ld = H;
  p.out_feats = H;
  p.w_perm = w_perm;
  p.a_scale = L->fp8 ? L->sc_dn : nullptr;
  p.a_codes = L->fp8 ? static_cast<const uint8_t*>(L->w_dn) : nullptr;
  if (f32) {
    // three terms of I_pad / 32 k-blocks; y fp32
    p.kb_term = Ip / moe::kBK32;
    p.num_kb = 3 * p.kb_term;
    p.out = nullptr;
    p.out_f32 = reinterpret_cast<float*>(ws + w.y);
    p.out_ld = H;
  }
  MOE_CUDA(f32       ? moe::launch_gemm_down_tf32(dn, p, L->num_sms, dn_blocks, st)
           : L->fp8  ? moe::launch_gemm_down_fp8(dn8, p, L->num_sms, dn_blocks, st)
           : pair_dn ? moe::launch_gemm_down_pair(dn, p, st)
                     : moe::launch_gemm_down(dn, p, L->num_sms, dn_blocks, st));
  MOE_CUDA(mark(6));
  if (f32)
    MOE_CUDA(moe::launch_combine_f32(reinterpret_cast<const float*>(ws + w.y), pos, T, k, H, xb,
                                     L->with_shared != 0, out, st));
  else
    MOE_CUDA(moe::launch_combine(ybuf, pos, T, k, H, xb, L->with_shared != 0, out, st));
  MOE_CUDA(mark(7));

  return copy_routing(routing, T, k, El, topk_idx, topk_w, counts, row_start, perm, st);
}

int moe_forward_host(moe_layer_t* L, const void* x_host, int T, void* out_host, void* workspace,
                     size_t ws_bytes, void* stream) {
  if (L == nullptr || T < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (x_host == nullptr || out_host == nullptr) return MOE_ERR_INVALID_ARG;
  size_t need = 0;
  int r = moe_workspace_size_host(L, T, &need);
  if (r != MOE_OK) return r;
  if (workspace == nullptr || ws_bytes < need || !aligned(workspace, 256)) return MOE_ERR_WORKSPACE;
  if (!L->loaded) return MOE_ERR_NOT_LOADED;
  DeviceGuard dg(L->device);
  if (!dg.ok) return MOE_ERR_CUDA;
  const size_t el = (L->cfg.act_dtype == MOE_BF16) ? 2 : 4;
  const size_t io_bytes = static_cast<size_t>(T) * L->cfg.hidden * el;
  const size_t base = ws_layout(L, T).total;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* x_dev = ws + base;
  void* out_dev = ws + base + align_up(io_bytes, kAlign);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MOE_CUDA(cudaMemcpyAsync(x_dev, x_host, io_bytes, cudaMemcpyHostToDevice, st));
  r = moe_forward(L, x_dev, T, out_dev, workspace, base, stream, nullptr);
  if (r != MOE_OK) return r;
  MOE_CUDA(cudaMemcpyAsync(out_host, out_dev, io_bytes, cudaMemcpyDeviceToHost, st));
  MOE_CUDA(cudaStreamSynchronize(st));
  return MOE_OK;
}

int moe_forward_host_async(moe_layer_t* L, const void* x_host, int T, void* out_host,
                           void* workspace, size_t ws_bytes, void* stream) {
  if (L == nullptr || T < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (x_host == nullptr || out_host == nullptr) return MOE_ERR_INVALID_ARG;
  size_t need = 0;
  int r = moe_workspace_size_host(L, T, &need);
  if (r != MOE_OK) return r;
  if (workspace == nullptr || ws_bytes < need || !aligned(workspace, 256)) return MOE_ERR_WORKSPACE;
  if (!L->loaded) return MOE_ERR_NOT_LOADED;
  DeviceGuard dg(L->device);
  if (!dg.ok) return MOE_ERR_CUDA;
  if (L->st_in == nullptr) {  // first call: the copy streams and the slot events
    MOE_CUDA(cudaStreamCreateWithFlags(&L->st_in, cudaStreamNonBlocking));
    MOE_CUDA(cudaStreamCreateWithFlags(&L->st_out, cudaStreamNonBlocking));
    for (int i = 0; i < 2; ++i) {
      MOE_CUDA(cudaEventCreateWithFlags(&L->ev_in[i], cudaEventDisableTiming));
      MOE_CUDA(cudaEventCreateWithFlags(&L->ev_fwd[i], cudaEventDisableTiming));
      MOE_CUDA(cudaEventCreateWithFlags(&L->ev_out[i], cudaEventDisableTiming));
    }
  }
  const size_t el = (L->cfg.act_dtype == MOE_BF16) ? 2 : 4;
  const size_t io_bytes = static_cast<size_t>(T) * L->cfg.hidden * el;
  const size_t io = align_up(io_bytes, kAlign);
  const size_t base = ws_layout(L, T).total;
  const int slot = static_cast<int>(L->host_calls & 1ull);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* x_dev = ws + base + slot * 2 * io;
  void* out_dev = ws + base + slot * 2 * io + io;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // a new T moves the staging slots: start after every earlier call is done
  if (L->host_calls > 0 && T != L->host_T)
    MOE_CUDA(cudaStreamWaitEvent(L->st_in, L->ev_out[(L->host_calls - 1ull) & 1ull], 0));
  L->host_T = T;
  // input: once the forward two calls back has read this slot's x
  MOE_CUDA(cudaStreamWaitEvent(L->st_in, L->ev_fwd[slot], 0));
  MOE_CUDA(cudaMemcpyAsync(x_dev, x_host, io_bytes, cudaMemcpyHostToDevice, L->st_in));
  MOE_CUDA(cudaEventRecord(L->ev_in[slot], L->st_in));
  // forward: after its input, and after the output copy two calls back has
  // read this slot's out
  MOE_CUDA(cudaStreamWaitEvent(st, L->ev_in[slot], 0));
  MOE_CUDA(cudaStreamWaitEvent(st, L->ev_out[slot], 0));
  r = moe_forward(L, x_dev, T, out_dev, workspace, base, stream, nullptr);
  if (r != MOE_OK) return r;
  MOE_CUDA(cudaEventRecord(L->ev_fwd[slot], st));
  // output
  MOE_CUDA(cudaStreamWaitEvent(L->st_out, L->ev_fwd[slot], 0));
  MOE_CUDA(cudaMemcpyAsync(out_host, out_dev, io_bytes, cudaMemcpyDeviceToHost, L->st_out));
  MOE_CUDA(cudaEventRecord(L->ev_out[slot], L->st_out));
  ++L->host_calls;
  return MOE_OK;
}

int moe_forward_host_join(moe_layer_t* L, void* stream) {
  if (L == nullptr) return MOE_ERR_INVALID_ARG;
  if (L->host_calls == 0) return MOE_OK;
  DeviceGuard dg(L->device);
  if (!dg.ok) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the last call's output copy follows every earlier one on the copy stream
  const int last = static_cast<int>((L->host_calls - 1ull) & 1ull);
  MOE_CUDA(cudaStreamWaitEvent(st, L->ev_out[last], 0));
  return MOE_OK;
}

int moe_get_device_error(moe_layer_t* L, int* device_err) {
  if (L == nullptr || device_err == nullptr) return MOE_ERR_INVALID_ARG;
  DeviceGuard dg(L->device);
  if (!dg.ok) return MOE_ERR_CUDA;
  int v = 0;
  MOE_CUDA(cudaDeviceSynchronize());
  MOE_CUDA(cudaMemcpy(&v, L->status, sizeof(int), cudaMemcpyDeviceToHost));
  MOE_CUDA(cudaMemset(L->status, 0, sizeof(int)));
  *device_err = v;
  return v == 0 ? MOE_OK : MOE_ERR_DEVICE_TIMEOUT;
}

int moe_check_fused_timeout(moe_layer_t* L, const void* x, int T, void* out, void* workspace,
                            size_t ws_bytes, int limit_us, int* device_status) {
  if (L == nullptr || x == nullptr || out == nullptr || x == out || limit_us <= 0 ||
      limit_us > 10000000)
    return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(out, 16)) return MOE_ERR_INVALID_ARG;
  if (!L->loaded) return MOE_ERR_NOT_LOADED;
  if (T <= 0 || T > kMaxTokens || !fused_eligible(L, T)) return MOE_ERR_UNSUPPORTED;
  const WsLayout w = ws_layout(L, T);
  if (workspace == nullptr || ws_bytes < w.total || !aligned(workspace, 256))
    return MOE_ERR_WORKSPACE;
  DeviceGuard dg(L->device);
  if (!dg.ok) return MOE_ERR_CUDA;
  MOE_CUDA(cudaDeviceSynchronize());
  MOE_CUDA(cudaMemset(L->status, 0, sizeof(int)));
  const int r = launch_fused_forward(L, x, T, out, static_cast<uint8_t*>(workspace), w, nullptr,
                                     nullptr, static_cast<uint64_t>(limit_us) * 1000ull, 1u);
  if (r != MOE_OK) return r;
  int v = 0;
  MOE_CUDA(cudaDeviceSynchronize());
  MOE_CUDA(cudaMemcpy(&v, L->status, sizeof(int), cudaMemcpyDeviceToHost));
  MOE_CUDA(cudaMemset(L->status, 0, sizeof(int)));
  if (device_status != nullptr) *device_status = v;
  return v == 1 ? MOE_OK : MOE_ERR_CUDA;  // exactly the timeout bit
}

int moe_set_path(moe_layer_t* L, int path) {
  if (L == nullptr || path < MOE_PATH_AUTO || path > MOE_PATH_FUSED) return MOE_ERR_INVALID_ARG;
  L->path = path;
  return MOE_OK;
}

int moe_forward_path(const moe_layer_t* L, int T) {
  if (L == nullptr || T <= 0) return 0;
  return forward_path(L, T);
}

int moe_kernel_launches(const moe_layer_t* L, int T) {
  if (L == nullptr || T <= 0) return 0;
  if (forward_path(L, T) == MOE_PATH_FUSED) return 1;
  // router, top-k, counting sort (one kernel up to kSortChunk tokens, else
  // three), gather, gate|up GEMM, down GEMM, combine; a shard also maps the
  // selection to its own expert ids
  const bool shard = L->E_loc != L->cfg.num_experts || L->first != 0;
  return (T <= moe::kSortChunk ? 7 : 9) + (shard ? 1 : 0);
}

namespace {
void free_events(moe_layer* L) {
  for (cudaEvent_t e : L->events) cudaEventDestroy(e);
  L->events.clear();
  L->timing_capacity = 0;
  L->timing_recorded = 0;
}
}  // namespace

int moe_set_stage_timing(moe_layer_t* L, int capacity) {
  if (L == nullptr || capacity < 0) return MOE_ERR_INVALID_ARG;
  DeviceGuard dg(L->device);
  if (!dg.ok) return MOE_ERR_CUDA;
  free_events(L);
  if (capacity == 0) return MOE_OK;
  const size_t n = static_cast<size_t>(capacity) * (MOE_NUM_STAGES + 1);
  L->events.resize(n, nullptr);
  for (size_t i = 0; i < n; ++i) {
    if (cudaEventCreate(&L->events[i]) != cudaSuccess) {
      L->events.resize(i);
      free_events(L);
      return MOE_ERR_CUDA;
    }
  }
  L->timing_capacity = capacity;
  L->timing_recorded = 0;
  return MOE_OK;
}

int moe_get_stage_times(moe_layer_t* L, float* ms, int n_stages, int* n_forwards) {
  if (L == nullptr || ms == nullptr || n_forwards == nullptr || n_stages < 0 ||
      n_stages > MOE_NUM_STAGES)
    return MOE_ERR_INVALID_ARG;
  DeviceGuard dg(L->device);
  if (!dg.ok) return MOE_ERR_CUDA;
  for (int i = 0; i < n_stages; ++i) ms[i] = 0.f;
  const int n = L->timing_recorded;
  for (int f = 0; f < n; ++f) {
    cudaEvent_t* ev = &L->events[static_cast<size_t>(f) * (MOE_NUM_STAGES + 1)];
    MOE_CUDA(cudaEventSynchronize(ev[MOE_NUM_STAGES]));
    for (int i = 0; i < n_stages; ++i) {
      float t = 0.f;
      MOE_CUDA(cudaEventElapsedTime(&t, ev[i], ev[i + 1]));
      ms[i] += t;
    }
  }
  *n_forwards = n;
  L->timing_recorded = 0;
  return MOE_OK;
}

void moe_destroy(moe_layer_t* L) {
  if (L == nullptr) return;
  {
    DeviceGuard dg(L->device);
    cudaDeviceSynchronize();
    free_events(L);
    if (L->st_in != nullptr) {
      for (int i = 0; i < 2; ++i) {
        cudaEventDestroy(L->ev_in[i]);
        cudaEventDestroy(L->ev_fwd[i]);
        cudaEventDestroy(L->ev_out[i]);
      }
      cudaStreamDestroy(L->st_in);
      cudaStreamDestroy(L->st_out);
    }
    cudaFree(L->w_gu);
    cudaFree(L->w_dn);
    cudaFree(L->sc_gu);
    cudaFree(L->sc_dn);
    cudaFree(L->router_w);
    cudaFree(L->router_b);
    cudaFree(L->router_tc);
    cudaFree(L->router_t);
    cudaFree(L->status);
  }
  delete L;
}

int moe_forward_oneshot(const void* x, const float* router_w, const float* router_bias,
                        const void* w_gate, const void* w_up, const void* w_down,
                        const void* sh_gate, const void* sh_up, const void* sh_down, int T, int H,
                        int E, int k, int I, float scale, float swiglu_limit,
                        float swiglu_limit_shared, int act_dtype, int weight_dtype, void* out,
                        void* stream) {
  moe_config_t c{};
  c.hidden = H;
  c.num_experts = E;
  c.top_k = k;
  c.intermediate = I;
  c.shared_intermediate = I;
  c.norm_expert_weight = 1;
  c.routed_scaling_factor = scale;
  c.use_router_bias = router_bias != nullptr ? 1 : 0;
  c.swiglu_limit = swiglu_limit;
  c.swiglu_limit_shared = swiglu_limit_shared;
  c.act_dtype = act_dtype;
  c.weight_dtype = weight_dtype;
  int r = moe_config_check(&c);
  if (r != MOE_OK) return r;
  if (weight_dtype == MOE_FP8_E4M3) return MOE_ERR_UNSUPPORTED;  // no scales in this list
  if (T < 0) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  moe_layer_t* L = nullptr;
  r = moe_create(&c, &L);
  if (r != MOE_OK) return r;
  r = moe_load_weights(L, router_w, router_bias, w_gate, w_up, w_down, sh_gate, sh_up, sh_down,
                       stream);
  void* ws = nullptr;
  size_t bytes = 0;
  if (r == MOE_OK) r = moe_workspace_size(L, T, &bytes);
  if (r == MOE_OK && cudaMalloc(&ws, bytes) != cudaSuccess) r = MOE_ERR_CUDA;
  if (r == MOE_OK) r = moe_forward(L, x, T, out, ws, bytes, stream, nullptr);
  if (r == MOE_OK && cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    r = MOE_ERR_CUDA;
  if (ws != nullptr) cudaFree(ws);
  moe_destroy(L);
  return r;
}

}  // extern "C"
