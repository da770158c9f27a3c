// The dense SwiGLU MLP of the model's first three decoder layers
// (sglang-jax issue #1367 "Support Step 3.5 Flash", section "Model
// configuration", MLP bullet: the first 3 layers are dense with intermediate
// 11264; llm-atlas "Step-3.5-Flash", table "Raw config fields",
// intermediate_size 11264), on the MoE layer's expert GEMMs run with one
// group of all T rows:
//   h   = silu(min(x.W_gate, L)) * clip(x.W_up, -L, L)   K5 (gate|up + SwiGLU)
//   out = h . W_down                                       K6 (down, weight 1)
// When the tiles of one token block cannot fill the GPU (decode-sized T):
// up to 128 tokens with H % 256 == 0, one persistent stream-K launch runs
// both GEMMs and their reductions (dense_streamk.cu); otherwise both GEMMs
// split K, each part writes raw fp32 accumulators and a reduction kernel sums
// the parts in fixed order (then applies the SwiGLU, or writes out).
// fp32 weights take the fp32 expert path at every T: the one-SM tf32 GEMMs
// over the two-term split of weights, x and h (tf32.cuh), h and the output
// fp32.  Declared in include/moe.h (moe_dense_*).
#include <math.h>
#include <string.h>

#include <new>

#include "api_util.h"
#include "dense_streamk.h"
#include "moe_internal.h"

struct moe_dense {
  moe_dense_config_t cfg;
  int device;
  int num_sms;
  int I_pad;
  __nv_bfloat16* w_gu;  // [2 * I_pad, H]: blocks of 128 gate rows then 128 up rows
  __nv_bfloat16* w_dn;  // [H, I_pad]
  int f32;              // fp32 weights: the fp32 path (w_gu32 / w_dn32 instead)
  float* w_gu32;        // [2 * I_pad, 2H]: the same rows as [hi | lo] fp32
  float* w_dn32;        // [H, 2 * I_pad]
  CUtensorMap tm_gu32;  // box 32 x 256
  CUtensorMap tm_dn32;  // box 32 x 128
  int* status;
  int loaded;
  // the one-launch stream-K forward (T <= 128): its running counters, with
  // the words from which each forward derives its targets (dense_streamk.cu)
  unsigned int* sk_cnt;
  CUtensorMap tm_gu;    // box 64 x 256 (one CTA per tile)
  CUtensorMap tm_gu128; // box 64 x 128 (split-K partial tiles)
  CUtensorMap tm_gu_pw; // CTA pairs, wide stages: 64 + 64 rows x 2 K blocks
  CUtensorMap tm_gu_pn; // CTA pairs, narrow stages: 64 + 64 rows x 3 K blocks
  CUtensorMap tm_dn;    // box 64 x 128
  CUtensorMap tm_dn_pw; // CTA pairs: 128 rows x 2 K blocks
  CUtensorMap tm_dn_pn; // CTA pairs: 128 rows x 3 K blocks
};

namespace {

constexpr int kMaxTokens = 1 << 20;
constexpr size_t kAlign = 1024;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

__global__ void cast_f32_bf16_kernel(const float* __restrict__ x, __nv_bfloat16* __restrict__ y,
                                     size_t n) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    y[i] = __float2bfloat16_rn(x[i]);
}

__global__ void cast_bf16_f32_kernel(const __nv_bfloat16* __restrict__ x, float* __restrict__ y,
                                     size_t n) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    y[i] = __bfloat162float(x[i]);
}

__global__ void fill_f32_kernel(float* __restrict__ p, float v, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) p[i] = v;
}

// h[t][f] = silu(min(a, L)) * clip(u, -L, L) with a, u the sums over the S
// split-K parts (in order) of packed rows (f / 128) * 256 + f % 128 (gate)
// and that + 128 (up); parts [S][T][2 * I_pad] fp32.
__global__ void swiglu_parts_kernel(const float* __restrict__ parts, int S, size_t part_stride,
                                    int T, int I_pad, float L, __nv_bfloat16* __restrict__ h) {
  const size_t n = static_cast<size_t>(T) * I_pad;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t t = i / I_pad;
    const int f = static_cast<int>(i % I_pad);
    const size_t gr = t * 2 * static_cast<size_t>(I_pad) + (f / 128) * 256 + f % 128;
    float a = 0.f, u = 0.f;
    for (int z = 0; z < S; ++z) {
      a += parts[z * part_stride + gr];
      u += parts[z * part_stride + gr + 128];
    }
    if (L > 0.f) {
      a = fminf(a, L);
      u = fminf(fmaxf(u, -L), L);
    }
    h[i] = __float2bfloat16_rn(a / (1.0f + __expf(-a)) * u);
  }
}

// out[i] = sum over the S parts (in order) of parts[z][i].
template <typename TO>
__global__ void sum_parts_kernel(const float* __restrict__ parts, int S, size_t part_stride,
                                 size_t n, TO* __restrict__ out) {
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    float v = 0.f;
    for (int z = 0; z < S; ++z) v += parts[z * part_stride + i];
    if constexpr (sizeof(TO) == 2)
      out[i] = __float2bfloat16_rn(v);
    else
      out[i] = v;
  }
}

// Split-K parts for a GEMM whose tiles (one token block) are too few for the
// GPU: the smallest divisor S of the k-block count (up to 16) that fills the
// SMs' waves to >= 85 %, else the best filling one; 1 when the tiles already
// fill the GPU.
int choose_parts(int tiles, int num_kb, int num_sms) {
  if (tiles >= num_sms) return 1;
  int best = 1;
  double best_eff = 0.0;
  for (int S = 1; S <= 16; ++S) {
    if (num_kb % S != 0 || num_kb / S < 2) continue;
    const int n = tiles * S;
    const double eff = static_cast<double>(n) / (((n + num_sms - 1) / num_sms) * num_sms);
    if (eff >= 0.85) return S;
    if (eff > best_eff + 1e-9) {
      best = S;
      best_eff = eff;
    }
  }
  return best;
}

unsigned grid_for(size_t n, int num_sms) {
  const size_t blocks = (n + 255) / 256;
  const size_t cap = static_cast<size_t>(num_sms) * 8;
  return static_cast<unsigned>(blocks < cap ? (blocks > 0 ? blocks : 1) : cap);
}

struct DenseWs {
  size_t xb, h, y, ones, parts, total;
  size_t xs, h32, y32;  // fp32 path: x and h as [hi | lo] rows, y fp32 (bf16 out)
  int s_gu, s_dn;  // split-K parts of the two GEMMs (1: no split)
  bool sk;         // the one-launch stream-K forward (sk_parts: its slots per pass)
  int sk_seg[moe::kSkPasses];
  size_t sk_parts[moe::kSkPasses];
};

// The one-launch stream-K forward serves decode-sized T when H splits into
// 256-row down tiles and the grid fits its reduction staging.
bool use_streamk(const moe_dense* L, int T) {
  return T <= moe::kSkMaxTokens && L->cfg.hidden % 256 == 0 && L->num_sms <= moe::kSkMaxGrid &&
         moe::dense_streamk_grid() == L->num_sms;
}

DenseWs dense_ws(const moe_dense* L, int T) {
  const size_t H = L->cfg.hidden;
  DenseWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes, kAlign);
    return at;
  };
  const bool xf = L->cfg.act_dtype == MOE_F32;
  if (L->f32) {  // the fp32 path: one-SM tf32 tiles at every T
    w.xs = take(static_cast<size_t>(T) * H * 8);
    w.h32 = take(static_cast<size_t>(T) * L->I_pad * 8);
    w.y32 = xf ? 0 : take(static_cast<size_t>(T) * H * 4);
    w.ones = take(static_cast<size_t>(T) * sizeof(float));
    w.s_gu = w.s_dn = 1;
    w.total = off;
    return w;
  }
  w.xb = xf ? take(static_cast<size_t>(T) * H * 2) : 0;    // bf16 copy of fp32 x
  w.h = take(static_cast<size_t>(T) * L->I_pad * 2);
  if (use_streamk(L, T)) {
    const size_t G = L->num_sms;
    moe::SkPass ps[moe::kSkPasses];
    moe::dense_streamk_passes(L->cfg.hidden, L->I_pad, ps);
    w.sk = true;
    w.s_gu = w.s_dn = 1;
    for (int q = 0; q < moe::kSkPasses; ++q) {
      w.sk_seg[q] = moe::dense_streamk_max_seg(ps[q].tiles, ps[q].nkb, static_cast<int>(G));
      w.sk_parts[q] = take(G * w.sk_seg[q] * T * 256 * sizeof(float));
    }
    w.total = off;
    return w;
  }
  w.y = xf ? take(static_cast<size_t>(T) * H * 2) : 0;     // bf16 result before widening
  w.ones = take(static_cast<size_t>(T) * sizeof(float));  // the down GEMM's row weights
  // split-K only below the CTA-pair range (one token block of tiles)
  const int Ip = L->I_pad;
  const int tok_blocks = (T + moe::kBN - 1) / moe::kBN;
  const bool small = T < moe::kPairMinTokens && (L->cfg.hidden / moe::kBM) % 2 == 0;
  w.s_gu = small ? choose_parts((Ip / moe::kBM) * tok_blocks, L->cfg.hidden / moe::kBK,
                                L->num_sms)
                 : 1;
  w.s_dn = small ? choose_parts((L->cfg.hidden / (2 * moe::kBM)) * tok_blocks, Ip / moe::kBK,
                                L->num_sms)
                 : 1;
  const size_t gu_parts = w.s_gu > 1 ? static_cast<size_t>(w.s_gu) * T * 2 * Ip : 0;
  const size_t dn_parts = w.s_dn > 1 ? static_cast<size_t>(w.s_dn) * T * H : 0;
  w.parts = take((gu_parts > dn_parts ? gu_parts : dn_parts) * sizeof(float));
  w.total = off;
  return w;
}

// The fp32 path's forward (L->f32): x split into [hi | lo] rows, gate|up
// and down on the one-SM tf32 kernels with one group of T rows, h fp32 as
// [hi | lo], the output fp32 (widened from fp32 y for a bf16 output).
int dense_forward_f32(moe_dense* L, const void* x, int T, void* out, uint8_t* ws,
                      const DenseWs& w, cudaStream_t st) {
  const int H = L->cfg.hidden, Ip = L->I_pad;
  const bool xf = L->cfg.act_dtype == MOE_F32;
  float* xs = reinterpret_cast<float*>(ws + w.xs);
  float* h32 = reinterpret_cast<float*>(ws + w.h32);
  float* y32 = xf ? static_cast<float*>(out) : reinterpret_cast<float*>(ws + w.y32);
  float* ones = reinterpret_cast<float*>(ws + w.ones);
  // the split rows of x: the gather with no routed rows and T identity rows
  MOE_CUDA(moe::launch_gather_split(x, !xf, nullptr, 0, 1, T, H, xs, L->num_sms, st));
  fill_f32_kernel<<<grid_for(static_cast<size_t>(T), L->num_sms), 256, 0, st>>>(ones, 1.f, T);
  MOE_CUDA(cudaGetLastError());
  moe::GemmMaps gu{}, dn{};
  gu.a = L->tm_gu32;
  dn.a = L->tm_dn32;
  if (!moe::encode_f32_2d(&gu.b, xs, T, 2 * H, moe::kBBoxRows) ||
      !moe::encode_f32_2d(&gu.bw, xs, T, 2 * H, moe::kBN) ||
      !moe::encode_f32_2d(&dn.b, h32, T, 2 * Ip, moe::kBBoxRows) ||
      !moe::encode_f32_2d(&dn.bw, h32, T, 2 * Ip, moe::kBN))
    return MOE_ERR_CUDA;
  gu.bsh = gu.b;
  gu.bshw = gu.bw;
  dn.bsh = dn.b;
  dn.bshw = dn.bw;
  moe::GemmParams p{};
  p.single_rows = T;
  p.G = 1;
  p.E = -1;  // no shared group
  p.k_parts = 1;
  p.status = L->status;
  p.limit = L->cfg.swiglu_limit;
  p.limit_shared = L->cfg.swiglu_limit;
  p.kb_term = H / moe::kBK32;
  p.num_kb = 3 * p.kb_term;
  p.m_tiles = Ip / moe::kBM;
  p.a_rows_per_group = 2 * Ip;
  p.out_f32 = h32;
  p.out_ld = 2 * Ip;
  p.out_feats = Ip;
  MOE_CUDA(moe::launch_gemm_gate_up_tf32(gu, p, L->num_sms, st));
  const int dn_blocks = moe::gemm_down_blocks(H);
  p.kb_term = Ip / moe::kBK32;
  p.num_kb = 3 * p.kb_term;
  p.m_tiles = H / moe::kBM / dn_blocks;
  p.a_rows_per_group = H;
  p.out_f32 = y32;
  p.out_ld = H;
  p.out_feats = H;
  p.w_perm = ones;
  MOE_CUDA(moe::launch_gemm_down_tf32(dn, p, L->num_sms, dn_blocks, st));
  if (!xf) {
    const size_t n = static_cast<size_t>(T) * H;
    cast_f32_bf16_kernel<<<grid_for(n, L->num_sms), 256, 0, st>>>(
        y32, static_cast<__nv_bfloat16*>(out), n);
    MOE_CUDA(cudaGetLastError());
  }
  return MOE_OK;
}

}  // namespace

extern "C" {

int moe_dense_config_check(const moe_dense_config_t* c) {
  if (c == nullptr) return MOE_ERR_INVALID_ARG;
  if (c->hidden <= 0 || c->intermediate <= 0) return MOE_ERR_INVALID_ARG;
  if ((c->act_dtype != MOE_F32 && c->act_dtype != MOE_BF16) ||
      (c->weight_dtype != MOE_F32 && c->weight_dtype != MOE_BF16 &&
       c->weight_dtype != MOE_FP8_E4M3))
    return MOE_ERR_INVALID_ARG;
  if (!isfinite(c->swiglu_limit) || c->swiglu_limit < 0.f) return MOE_ERR_INVALID_ARG;
  if (c->weight_dtype == MOE_FP8_E4M3) return MOE_ERR_UNSUPPORTED;
  if (c->hidden % 128 != 0 || c->hidden > 16384 || c->intermediate > 32768)
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

int moe_dense_create(const moe_dense_config_t* cfg, moe_dense_t** out) {
  if (out == nullptr) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  const int chk = moe_dense_config_check(cfg);
  if (chk != MOE_OK) return chk;
  moe_dense* L = new (std::nothrow) moe_dense();
  if (L == nullptr) return MOE_ERR_CUDA;
  L->cfg = *cfg;
  L->I_pad = (cfg->intermediate + 127) / 128 * 128;
  L->f32 = cfg->weight_dtype == MOE_F32 ? 1 : 0;
  if (cudaGetDevice(&L->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&L->num_sms, cudaDevAttrMultiProcessorCount, L->device) !=
          cudaSuccess) {
    delete L;
    return MOE_ERR_CUDA;
  }
  const size_t H = cfg->hidden, Ip = L->I_pad;
  if (L->f32) {
    if (moe::gemm_configure_device() != cudaSuccess ||
        cudaMalloc(&L->w_gu32, 2 * Ip * H * 8) != cudaSuccess ||
        cudaMalloc(&L->w_dn32, H * Ip * 8) != cudaSuccess ||
        cudaMalloc(&L->status, sizeof(int)) != cudaSuccess ||
        cudaMemset(L->status, 0, sizeof(int)) != cudaSuccess ||
        !moe::encode_f32_2d(&L->tm_gu32, L->w_gu32, 2 * Ip, 2 * H, 2 * moe::kBM) ||
        !moe::encode_f32_2d(&L->tm_dn32, L->w_dn32, H, 2 * Ip, moe::kBM)) {
      moe_dense_destroy(L);
      return MOE_ERR_CUDA;
    }
    *out = L;
    return MOE_OK;
  }
  if (moe::gemm_configure_device() != cudaSuccess ||
      moe::gemm_pair_configure_device(L->num_sms) != cudaSuccess ||
      moe::dense_streamk_configure_device(L->num_sms) != cudaSuccess ||
      cudaMalloc(&L->w_gu, 2 * Ip * H * 2) != cudaSuccess ||
      cudaMalloc(&L->w_dn, H * Ip * 2) != cudaSuccess ||
      cudaMalloc(&L->status, sizeof(int)) != cudaSuccess ||
      cudaMemset(L->status, 0, sizeof(int)) != cudaSuccess ||
      cudaMalloc(&L->sk_cnt, moe::dense_streamk_counters(cfg->hidden, L->I_pad) * 4) !=
          cudaSuccess ||
      cudaMemset(L->sk_cnt, 0, moe::dense_streamk_counters(cfg->hidden, L->I_pad) * 4) !=
          cudaSuccess ||
      !moe::encode_bf16_2d(&L->tm_gu, L->w_gu, 2 * Ip, H, 2 * moe::kBM) ||
      !moe::encode_bf16_2d(&L->tm_gu128, L->w_gu, 2 * Ip, H, moe::kBM) ||
      !moe::encode_bf16_gate_up_pair(&L->tm_gu_pw, L->w_gu, 2 * Ip, H, 2) ||
      !moe::encode_bf16_gate_up_pair(&L->tm_gu_pn, L->w_gu, 2 * Ip, H, 3) ||
      !moe::encode_bf16_2d(&L->tm_dn, L->w_dn, H, Ip, moe::kBM) ||
      !moe::encode_bf16_kblocks(&L->tm_dn_pw, L->w_dn, H, Ip, moe::kBM, 2) ||
      !moe::encode_bf16_kblocks(&L->tm_dn_pn, L->w_dn, H, Ip, moe::kBM, 3)) {
    moe_dense_destroy(L);
    return MOE_ERR_CUDA;
  }
  *out = L;
  return MOE_OK;
}

int moe_dense_load_weights(moe_dense_t* L, const void* w_gate, const void* w_up,
                           const void* w_down, void* stream) {
  if (L == nullptr || w_gate == nullptr || w_up == nullptr || w_down == nullptr)
    return MOE_ERR_INVALID_ARG;
  moe::DeviceGuard dg(L->device);
  if (!dg.ok) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int H = L->cfg.hidden, I = L->cfg.intermediate, Ip = L->I_pad;
  const bool wb = L->cfg.weight_dtype == MOE_BF16;
  if (L->f32) {
    MOE_CUDA(cudaMemsetAsync(L->w_gu32, 0, static_cast<size_t>(2) * Ip * H * 8, st));
    MOE_CUDA(cudaMemsetAsync(L->w_dn32, 0, static_cast<size_t>(H) * Ip * 8, st));
    MOE_CUDA(moe::launch_pack_gate_up_split(w_gate, false, 1, H, I, Ip, 0, L->w_gu32, st));
    MOE_CUDA(moe::launch_pack_gate_up_split(w_up, false, 1, H, I, Ip, 1, L->w_gu32, st));
    MOE_CUDA(moe::launch_pack_down_split(w_down, false, 1, H, I, Ip, L->w_dn32, st));
    L->loaded = 1;
    return MOE_OK;
  }
  MOE_CUDA(cudaMemsetAsync(L->w_gu, 0, static_cast<size_t>(2) * Ip * H * 2, st));
  MOE_CUDA(cudaMemsetAsync(L->w_dn, 0, static_cast<size_t>(H) * Ip * 2, st));
  MOE_CUDA(moe::launch_pack_gate_up(w_gate, wb, 1, H, I, Ip, 0, L->w_gu, st));
  MOE_CUDA(moe::launch_pack_gate_up(w_up, wb, 1, H, I, Ip, 1, L->w_gu, st));
  MOE_CUDA(moe::launch_pack_down(w_down, wb, 1, H, I, Ip, L->w_dn, st));
  L->loaded = 1;
  return MOE_OK;
}

int moe_dense_workspace_size(const moe_dense_t* L, int T, size_t* bytes) {
  if (L == nullptr || bytes == nullptr || T < 0) return MOE_ERR_INVALID_ARG;
  if (T > kMaxTokens) return MOE_ERR_UNSUPPORTED;
  *bytes = T == 0 ? 0 : dense_ws(L, T).total;
  return MOE_OK;
}

int moe_dense_forward(moe_dense_t* L, const void* x, int T, void* out, void* workspace,
                      size_t ws_bytes, void* stream) {
  if (L == nullptr || T < 0) return MOE_ERR_INVALID_ARG;
  if (T > kMaxTokens) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (x == nullptr || out == nullptr || x == out) return MOE_ERR_INVALID_ARG;
  if (!moe::aligned(x, 16) || !moe::aligned(out, 16)) return MOE_ERR_INVALID_ARG;
  if (!L->loaded) return MOE_ERR_NOT_LOADED;
  const DenseWs w = dense_ws(L, T);
  if (workspace == nullptr || ws_bytes < w.total || !moe::aligned(workspace, 256))
    return MOE_ERR_WORKSPACE;
  moe::DeviceGuard dg(L->device);
  if (!dg.ok) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int H = L->cfg.hidden, Ip = L->I_pad;
  const bool xf = L->cfg.act_dtype == MOE_F32;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t n = static_cast<size_t>(T) * H;
  if (L->f32) return dense_forward_f32(L, x, T, out, ws, w, st);
  // bf16 operand rows (x itself when bf16)
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  if (xf) {
    __nv_bfloat16* xc = reinterpret_cast<__nv_bfloat16*>(ws + w.xb);
    cast_f32_bf16_kernel<<<grid_for(n, L->num_sms), 256, 0, st>>>(static_cast<const float*>(x),
                                                                    xc, n);
    MOE_CUDA(cudaGetLastError());
    xb = xc;
  }
  __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(ws + w.h);
  __nv_bfloat16* y = xf ? reinterpret_cast<__nv_bfloat16*>(ws + w.y)
                        : static_cast<__nv_bfloat16*>(out);
  if (w.sk) {  // decode-sized T: both GEMMs and their reductions in one launch
    moe::DenseStreamK d{};
    d.tm_gu = L->tm_gu128;
    d.tm_dn = L->tm_dn;
    const uint32_t n_mma = static_cast<uint32_t>((T + 15) & ~15);
    if (!moe::encode_bf16_2d(&d.tm_x, xb, T, H, n_mma) ||
        !moe::encode_bf16_2d(&d.tm_h, h, T, Ip, n_mma))
      return MOE_ERR_CUDA;
    d.T = T;
    d.H = H;
    d.I_pad = Ip;
    for (int q = 0; q < moe::kSkPasses; ++q) {
      d.max_seg[q] = w.sk_seg[q];
      d.parts[q] = reinterpret_cast<float*>(ws + w.sk_parts[q]);
    }
    d.limit = L->cfg.swiglu_limit;
    d.h = h;
    d.out = out;
    d.out_f32 = xf;
    d.counters = L->sk_cnt;
    d.status = L->status;
    MOE_CUDA(moe::launch_dense_streamk(d, st));
    return MOE_OK;
  }
  float* ones = reinterpret_cast<float*>(ws + w.ones);
  if (w.s_dn <= 1) {  // the unsplit down GEMM's row weights
    fill_f32_kernel<<<grid_for(static_cast<size_t>(T), L->num_sms), 256, 0, st>>>(ones, 1.f, T);
    MOE_CUDA(cudaGetLastError());
  }

  // one group of all T rows; CTA pairs (256-token tiles) from kPairMinTokens
  const bool pair = T >= moe::kPairMinTokens;
  const bool pair_dn = pair && (H / moe::kBM) % 2 == 0;
  const int dn_blocks = moe::gemm_down_blocks(H);
  moe::GemmMaps gu{}, dn{};
  if (pair) {  // CTA pairs: K-block maps (see launch_gemm_gate_up_pair)
    gu.a = L->tm_gu_pw;
    gu.a2 = L->tm_gu_pn;
    if (!moe::encode_bf16_kblocks(&gu.b, xb, T, H, moe::kBBoxRows, 3) ||
        !moe::encode_bf16_kblocks(&gu.bw, xb, T, H, moe::kBN, 2))
      return MOE_ERR_CUDA;
  } else {
    gu.a = L->tm_gu;
    if (!moe::encode_bf16_2d(&gu.b, xb, T, H, moe::kBBoxRows) ||
        !moe::encode_bf16_2d(&gu.bw, xb, T, H, moe::kBN))
      return MOE_ERR_CUDA;
  }
  if (pair_dn) {
    dn.a = L->tm_dn_pw;
    dn.a2 = L->tm_dn_pn;
    if (!moe::encode_bf16_kblocks(&dn.b, h, T, Ip, moe::kBBoxRows, 3) ||
        !moe::encode_bf16_kblocks(&dn.bw, h, T, Ip, moe::kBN, 2))
      return MOE_ERR_CUDA;
  } else {
    dn.a = L->tm_dn;
    if (!moe::encode_bf16_2d(&dn.b, h, T, Ip, moe::kBBoxRows) ||
        !moe::encode_bf16_2d(&dn.bw, h, T, Ip, moe::kBN))
      return MOE_ERR_CUDA;
  }
  if (!moe::encode_bf16_store(&gu.out, h, T, Ip) || !moe::encode_bf16_store(&dn.out, y, T, H))
    return MOE_ERR_CUDA;
  gu.bsh = gu.b;
  gu.bshw = gu.bw;
  dn.bsh = dn.b;
  dn.bshw = dn.bw;

  moe::GemmParams p{};
  p.single_rows = T;
  p.G = 1;
  p.E = -1;  // no shared group
  p.k_parts = 1;
  p.status = L->status;
  p.limit = L->cfg.swiglu_limit;
  p.limit_shared = L->cfg.swiglu_limit;
  float* parts = reinterpret_cast<float*>(ws + w.parts);
  const int sgrid = L->num_sms;

  if (w.s_gu > 1) {
    // gate|up in S parts of K: raw accumulators of all 2 * I_pad packed rows
    moe::GemmMaps pg = gu;
    pg.a = L->tm_gu128;
    p.k_parts = w.s_gu;
    p.num_kb = H / moe::kBK / w.s_gu;
    p.m_tiles = 2 * Ip / (2 * moe::kBM);
    p.a_rows_per_group = 2 * Ip;
    p.out_f32 = parts;
    p.out_ld = 2 * Ip;
    p.out_feats = 2 * Ip;
    p.part_stride = static_cast<size_t>(T) * 2 * Ip;
    MOE_CUDA(moe::launch_gemm_partial(pg, p, sgrid, st));
    swiglu_parts_kernel<<<grid_for(static_cast<size_t>(T) * Ip, L->num_sms), 256, 0, st>>>(
        parts, w.s_gu, p.part_stride, T, Ip, L->cfg.swiglu_limit, h);
    MOE_CUDA(cudaGetLastError());
  }
  if (w.s_dn > 1) {
    if (w.s_gu <= 1) {  // gate|up unsplit
      p.k_parts = 1;
      p.num_kb = H / moe::kBK;
      p.m_tiles = Ip / moe::kBM;
      p.a_rows_per_group = 2 * Ip;
      p.out = h;
      p.out_ld = Ip;
      p.out_feats = Ip;
      MOE_CUDA(moe::launch_gemm_gate_up(gu, p, L->num_sms, st));
    }
    // down in S parts of K, then the sum in order
    p.k_parts = w.s_dn;
    p.num_kb = Ip / moe::kBK / w.s_dn;
    p.m_tiles = H / (2 * moe::kBM);
    p.a_rows_per_group = H;
    p.out_f32 = parts;
    p.out_ld = H;
    p.out_feats = H;
    p.part_stride = static_cast<size_t>(T) * H;
    MOE_CUDA(moe::launch_gemm_partial(dn, p, sgrid, st));
    if (xf)
      sum_parts_kernel<float><<<grid_for(n, L->num_sms), 256, 0, st>>>(
          parts, w.s_dn, p.part_stride, n, static_cast<float*>(out));
    else
      sum_parts_kernel<__nv_bfloat16><<<grid_for(n, L->num_sms), 256, 0, st>>>(
          parts, w.s_dn, p.part_stride, n, static_cast<__nv_bfloat16*>(out));
    MOE_CUDA(cudaGetLastError());
    return MOE_OK;
  }
  if (w.s_gu > 1) {  // down unsplit after a split gate|up
    p.k_parts = 1;
    p.num_kb = Ip / moe::kBK;
    p.m_tiles = H / moe::kBM / dn_blocks;
    p.a_rows_per_group = H;
    p.out = y;
    p.out_ld = H;
    p.out_feats = H;
    p.w_perm = ones;
    MOE_CUDA(moe::launch_gemm_down(dn, p, L->num_sms, dn_blocks, st));
    if (xf) {
      cast_bf16_f32_kernel<<<grid_for(n, L->num_sms), 256, 0, st>>>(y, static_cast<float*>(out),
                                                                     n);
      MOE_CUDA(cudaGetLastError());
    }
    return MOE_OK;
  }

  p.num_kb = H / moe::kBK;
  p.m_tiles = Ip / moe::kBM;
  p.a_rows_per_group = 2 * Ip;
  p.out = h;
  p.out_ld = Ip;
  p.out_feats = Ip;
  MOE_CUDA(pair ? moe::launch_gemm_gate_up_pair(gu, p, st)
                : moe::launch_gemm_gate_up(gu, p, L->num_sms, st));

  p.num_kb = Ip / moe::kBK;
  p.m_tiles = pair_dn ? H / (2 * moe::kBM) : H / moe::kBM / dn_blocks;
  p.a_rows_per_group = H;
  p.out = y;
  p.out_ld = H;
  p.out_feats = H;
  p.w_perm = ones;
  MOE_CUDA(pair_dn ? moe::launch_gemm_down_pair(dn, p, st)
                   : moe::launch_gemm_down(dn, p, L->num_sms, dn_blocks, st));
  if (xf) {
    cast_bf16_f32_kernel<<<grid_for(n, L->num_sms), 256, 0, st>>>(y, static_cast<float*>(out), n);
    MOE_CUDA(cudaGetLastError());
  }
  return MOE_OK;
}

int moe_dense_get_device_error(moe_dense_t* L, int* device_err) {
  if (L == nullptr || device_err == nullptr) return MOE_ERR_INVALID_ARG;
  moe::DeviceGuard dg(L->device);
  if (!dg.ok) return MOE_ERR_CUDA;
  int v = 0;
  MOE_CUDA(cudaDeviceSynchronize());
  MOE_CUDA(cudaMemcpy(&v, L->status, sizeof(int), cudaMemcpyDeviceToHost));
  MOE_CUDA(cudaMemset(L->status, 0, sizeof(int)));
  if (v != 0 && L->sk_cnt != nullptr) {  // an aborted stream-K forward leaves its counters
                                         // short of their targets
    MOE_CUDA(cudaMemset(L->sk_cnt, 0,
                        moe::dense_streamk_counters(L->cfg.hidden, L->I_pad) * sizeof(unsigned int)));
  }
  *device_err = v;
  return v == 0 ? MOE_OK : MOE_ERR_DEVICE_TIMEOUT;
}

void moe_dense_destroy(moe_dense_t* L) {
  if (L == nullptr) return;
  {
    moe::DeviceGuard dg(L->device);
    cudaDeviceSynchronize();
    cudaFree(L->w_gu);
    cudaFree(L->w_dn);
    cudaFree(L->w_gu32);
    cudaFree(L->w_dn32);
    cudaFree(L->status);
    cudaFree(L->sk_cnt);
  }
  delete L;
}

}  // extern "C"
