// K3: deterministic token-to-expert grouping (histogram, scan, stable scatter)
// and K4: gather of the input rows into expert-contiguous order.
//
// The grouped matmul of an expert-parallel MoE ("EPMoE", sglang-jax issue
// #1367 "Support Step 3.5 Flash", sections "Reuse map" and "Implementation
// strategy") needs each expert's rows contiguous.  Definition kept here:
// perm lists the pair ids t * k + j of expert 0, then expert 1, ..., each in
// ascending t; pos[t * k + j] is the pair's slot in perm.  The shared expert
// is group E with the T identity rows [T*k, T*k + T) (or no rows).
//
// Expert shards: the caller passes local expert ids (another shard's expert
// is -1); such pairs get pos = -1 and no slot, the routed rows then end
// before T*k, and the shared group still starts at row T*k.
//
// No order-dependent atomics: each block owns kSortChunk tokens and records,
// per expert, a 128-bit mask of its tokens that chose that expert (atomicOr
// gives the same mask in any order).  A pair's rank inside its block is the
// popcount of the mask bits below its token, so the scatter is stable and
// bit-reproducible.
#include "moe_internal.h"
#include "tf32.cuh"
#include "moe_ptx.cuh"
#include "sort_device.cuh"

namespace moe {

namespace {

using sort::chunk_rank;
using sort::kMaskWords;
using sort::scan_groups;

__global__ void __launch_bounds__(256) sort_hist_kernel(const int* __restrict__ topk_idx, int T,
                                                        int k, int E, uint32_t* __restrict__ masks,
                                                        int* __restrict__ chunk_cnt) {
  pdl_wait();  // the previous kernel's results are visible
  extern __shared__ uint32_t sm[];
  sort::hist_chunk(blockIdx.x, topk_idx, T, k, E, masks, chunk_cnt, sm);
}

// One block: per expert, running offsets of the chunks; then the prefixes
// over the groups.
__global__ void __launch_bounds__(1024) sort_scan_kernel(
    const int* __restrict__ chunk_cnt, int nch, int T, int k, int E, int shared_rows, int bn_gu,
    int bn_dn, int mt_gu, int mt_dn, int* __restrict__ chunk_base, int* __restrict__ counts,
    int* __restrict__ row_start, int* __restrict__ tiles_gu, int* __restrict__ tiles_dn) {
  pdl_wait();  // the previous kernel's results are visible
  __shared__ int cnt_s[1025];
  sort::scan_block(chunk_cnt, nch, T, k, E, shared_rows, bn_gu, bn_dn, mt_gu, mt_dn, chunk_base,
                   counts, row_start, tiles_gu, tiles_dn, cnt_s);
}

// T <= kSortChunk (decode): histogram, prefixes and stable scatter in one block.
__global__ void __launch_bounds__(1024) sort_small_kernel(
    const int* __restrict__ topk_idx, const float* __restrict__ topk_w, int T, int k, int E,
    int shared_rows, int bn_gu, int bn_dn, int mt_gu, int mt_dn, int* __restrict__ counts,
    int* __restrict__ row_start,
    int* __restrict__ tiles_gu, int* __restrict__ tiles_dn, int* __restrict__ perm,
    int* __restrict__ pos, float* __restrict__ w_perm) {
  pdl_wait();  // the previous kernel's results are visible
  extern __shared__ uint32_t sm[];
  uint32_t* masks = sm;                                   // [E][4]
  int* cnt_s = reinterpret_cast<int*>(sm + E * kMaskWords);  // [E + 1]
  int* start_s = cnt_s + (E + 1);                         // [E + 1]
  for (int i = threadIdx.x; i < E * kMaskWords; i += blockDim.x) masks[i] = 0u;
  __syncthreads();
  for (int p = threadIdx.x; p < T * k; p += blockDim.x) {
    const int tl = p / k;
    const int e = topk_idx[p];
    if (static_cast<unsigned>(e) < static_cast<unsigned>(E))
      atomicOr(&masks[e * kMaskWords + (tl >> 5)], 1u << (tl & 31));
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int n = 0;
#pragma unroll
    for (int q = 0; q < kMaskWords; ++q) n += __popc(masks[e * kMaskWords + q]);
    cnt_s[e] = n;
  }
  if (threadIdx.x == 0) cnt_s[E] = shared_rows;
  __syncthreads();
  if (threadIdx.x < 32)
    scan_groups(cnt_s, E + 1, bn_gu, bn_dn, mt_gu, mt_dn, T * k, counts, row_start, tiles_gu,
                tiles_dn, start_s);
  __syncthreads();
  for (int p = threadIdx.x; p < T * k; p += blockDim.x) {
    const int tl = p / k;
    const int e = topk_idx[p];
    if (static_cast<unsigned>(e) >= static_cast<unsigned>(E)) {  // another shard's expert
      pos[p] = -1;
      continue;
    }
    const int slot = start_s[e] + chunk_rank(masks + e * kMaskWords, tl);
    perm[slot] = p;
    pos[p] = slot;
    w_perm[slot] = topk_w[p];
  }
  for (int t = threadIdx.x; t < T; t += blockDim.x) w_perm[T * k + t] = 1.0f;
}

__global__ void __launch_bounds__(256) sort_scatter_kernel(
    const int* __restrict__ topk_idx, const float* __restrict__ topk_w, int T, int k, int E,
    const uint32_t* __restrict__ masks, const int* __restrict__ chunk_base,
    const int* __restrict__ row_start, int* __restrict__ perm, int* __restrict__ pos,
    float* __restrict__ w_perm) {
  pdl_wait();  // the previous kernel's results are visible
  extern __shared__ uint32_t sm[];
  sort::scatter_chunk(blockIdx.x, topk_idx, topk_w, T, k, E, masks, chunk_base, row_start, perm,
                      pos, w_perm, sm);
}

__device__ __forceinline__ uint4 load8_bf16(const __nv_bfloat16* p) {
  return *reinterpret_cast<const uint4*>(p);
}

__device__ __forceinline__ uint4 load8_bf16(const float* p) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  uint4 q;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&q);
  h[0] = __floats2bfloat162_rn(a.x, a.y);
  h[1] = __floats2bfloat162_rn(a.z, a.w);
  h[2] = __floats2bfloat162_rn(b.x, b.y);
  h[3] = __floats2bfloat162_rn(b.z, b.w);
  return q;
}

// One warp per destination row, 16-byte vectors.  Rows [0, rows_routed) take
// x[perm[r] / k]; with write_shared, rows [rows_routed, rows_routed + T) take
// x[r - rows_routed] (the shared expert's rows, needed when x is fp32).
template <typename TX>
__global__ void __launch_bounds__(256) gather_kernel(const TX* __restrict__ x,
                                                     const int* __restrict__ perm,
                                                     int rows_routed, int k, int T, int H,
                                                     int write_shared,
                                                     __nv_bfloat16* __restrict__ xp) {
  pdl_wait();  // the previous kernel's results are visible
  const int lane = threadIdx.x & 31;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const int nrows = rows_routed + (write_shared ? T : 0);
  const int nvec = H / 8;
  for (int r = warp; r < nrows; r += nwarps) {
    const int t = (r < rows_routed) ? perm[r] / k : r - rows_routed;
    uint4* dst = reinterpret_cast<uint4*>(xp + static_cast<size_t>(r) * H);
    if (static_cast<unsigned>(t) >= static_cast<unsigned>(T)) {
      for (int v = lane; v < nvec; v += 32) dst[v] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const TX* src = x + static_cast<size_t>(t) * H;
    for (int v = lane; v < nvec; v += 32) dst[v] = load8_bf16(src + v * 8);
  }
}

__device__ __forceinline__ float to_float(float v) { return v; }
__device__ __forceinline__ float to_float(__nv_bfloat16 v) { return __bfloat162float(v); }

// The fp32 expert path's x_perm: row r = [x_hi | x_lo] of its token (the tf32
// split, 2H fp32), rows [0, rows_routed) from x[perm[r] / k], then the shared
// expert's rows [rows_routed, rows_routed + T) from x[r - rows_routed].  One
// warp per row, four values per lane step.
template <typename TX>
__global__ void __launch_bounds__(256) gather_split_kernel(const TX* __restrict__ x,
                                                           const int* __restrict__ perm,
                                                           int rows_routed, int k, int T, int H,
                                                           float* __restrict__ xp) {
  pdl_wait();  // the previous kernel's results are visible
  const int lane = threadIdx.x & 31;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const int nrows = rows_routed + T;
  const int nvec = H / 4;
  for (int r = warp; r < nrows; r += nwarps) {
    const int t = (r < rows_routed) ? perm[r] / k : r - rows_routed;
    float4* hi = reinterpret_cast<float4*>(xp + static_cast<size_t>(r) * 2 * H);
    float4* lo = hi + nvec;
    if (static_cast<unsigned>(t) >= static_cast<unsigned>(T)) {
      for (int v = lane; v < nvec; v += 32) hi[v] = lo[v] = make_float4(0.f, 0.f, 0.f, 0.f);
      continue;
    }
    const TX* src = x + static_cast<size_t>(t) * H;
    for (int v = lane; v < nvec; v += 32) {
      float f[4], a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        f[i] = to_float(src[4 * v + i]);
        tf32_split(f[i], a[i], b[i]);
      }
      hi[v] = make_float4(a[0], a[1], a[2], a[3]);
      lo[v] = make_float4(b[0], b[1], b[2], b[3]);
    }
  }
}

// Batches from which the bf16 gather runs per token with bulk copies (below,
// the row-per-warp form spreads a small batch over more SMs).
constexpr int kGatherRowsMinTokens = 1024;

// bf16 x: one warp per token at a time, its lane 0 issuing bulk (TMA) copies:
// the token's row is read into shared memory once and written to its k rows
// of x_perm (pos[t, j]) by k bulk stores.  Two row buffers per warp, so the
// next token's load overlaps this token's stores.
__global__ void __launch_bounds__(256) gather_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                          const int* __restrict__ pos, int T,
                                                          int k, int H,
                                                          __nv_bfloat16* __restrict__ xp,
                                                          int* status) {
  extern __shared__ __align__(128) uint8_t gsm[];
  pdl_wait();  // the previous kernel's results are visible
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int wpb = blockDim.x >> 5;
  const uint32_t row_bytes = static_cast<uint32_t>(H) * 2;
  const uint32_t buf0 = smem_u32(gsm) + static_cast<uint32_t>(warp) * 2 * row_bytes;
  const uint32_t bar0 = smem_u32(gsm) + static_cast<uint32_t>(wpb) * 2 * row_bytes + warp * 16;
  if (lane != 0) return;
  mbar_init(bar0, 1);
  mbar_init(bar0 + 8, 1);
  fence_mbar_init();
  uint32_t i = 0;
  for (int t = blockIdx.x * wpb + warp; t < T; t += gridDim.x * wpb, ++i) {
    const uint32_t b = i & 1u;
    const uint32_t buf = buf0 + b * row_bytes;
    const uint32_t bar = bar0 + 8 * b;
    int rows[32];
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < k) rows[j] = pos[static_cast<size_t>(t) * k + j];
    if (i >= 2) bulk_wait_group_read<1>();  // the stores that read this buffer are done with it
    mbar_arrive_expect_tx(bar, row_bytes);
    bulk_load_1d(buf, x + static_cast<size_t>(t) * H, row_bytes, bar);
    if (!mbar_wait(bar, (i >> 1) & 1u, nullptr, status)) break;
#pragma unroll
    for (int j = 0; j < 32; ++j)  // (pos -1: another shard's expert, no row)
      if (j < k && rows[j] >= 0) bulk_store_1d(xp + static_cast<size_t>(rows[j]) * H, buf, row_bytes);
    bulk_commit_group();
  }
  bulk_wait_group_all();
}

// Expert shard: global expert ids -> local ids (e - first for the shard's
// experts [first, first + count), else -1).
__global__ void localize_kernel(const int* __restrict__ topk_idx, int n, int first, int count,
                                int* __restrict__ local_idx) {
  pdl_wait();  // the previous kernel's results are visible
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int e = topk_idx[i] - first;
    local_idx[i] = static_cast<unsigned>(e) < static_cast<unsigned>(count) ? e : -1;
  }
}

}  // namespace

cudaError_t launch_localize(const int* topk_idx, int n, int first, int count, int* local_idx,
                            cudaStream_t st) {
  const int blocks = max(1, min((n + 255) / 256, 1024));
  return launch_pdl(localize_kernel, dim3(blocks), dim3(256), 0, st, topk_idx, n, first, count,
                    local_idx);
}

cudaError_t gather_configure_device() {
  return cudaFuncSetAttribute(gather_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              100 * 1024);
}

cudaError_t launch_sort(const int* topk_idx, const float* topk_w, int T, int k, int E,
                        int shared_rows, int bn_gu, int bn_dn, int m_tiles_gu, int m_tiles_dn,
                        uint32_t* masks, int* chunk_cnt, int* chunk_base, int* counts,
                        int* row_start, int* tiles_gu, int* tiles_dn, int* perm, int* pos,
                        float* w_perm, cudaStream_t st) {
  const int nch = (T + kSortChunk - 1) / kSortChunk;
  const size_t smem = static_cast<size_t>(E) * kMaskWords * sizeof(uint32_t);
  if (nch == 1) {
    const size_t smem1 = smem + 2 * static_cast<size_t>(E + 1) * sizeof(int);
    return launch_pdl(sort_small_kernel, dim3(1), dim3(1024), smem1, st, topk_idx, topk_w, T, k, E,
                      shared_rows, bn_gu, bn_dn, m_tiles_gu, m_tiles_dn, counts, row_start,
                      tiles_gu, tiles_dn, perm, pos, w_perm);
  }
  cudaError_t err = launch_pdl(sort_hist_kernel, dim3(nch), dim3(256), smem, st, topk_idx, T, k, E,
                               masks, chunk_cnt);
  if (err != cudaSuccess) return err;
  err = launch_pdl(sort_scan_kernel, dim3(1), dim3(1024), 0, st, chunk_cnt, nch, T, k, E,
                   shared_rows, bn_gu, bn_dn, m_tiles_gu, m_tiles_dn, chunk_base, counts,
                   row_start, tiles_gu, tiles_dn);
  if (err != cudaSuccess) return err;
  return launch_pdl(sort_scatter_kernel, dim3(nch), dim3(256), smem, st, topk_idx, topk_w, T, k, E,
                    masks, chunk_base, row_start, perm, pos, w_perm);
}

cudaError_t launch_gather_split(const void* x, bool x_bf16, const int* perm, int rows_routed,
                                int k, int T, int H, float* x_perm, int num_sms,
                                cudaStream_t st) {
  const int want = (rows_routed + T + 7) / 8;
  const int blocks = max(1, min(want, num_sms * 8));
  if (x_bf16)
    return launch_pdl(gather_split_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, st,
                      static_cast<const __nv_bfloat16*>(x), perm, rows_routed, k, T, H, x_perm);
  return launch_pdl(gather_split_kernel<float>, dim3(blocks), dim3(256), 0, st,
                    static_cast<const float*>(x), perm, rows_routed, k, T, H, x_perm);
}

cudaError_t launch_gather(const void* x, bool x_bf16, const int* perm, const int* pos,
                          int rows_routed, int k, int T, int H, bool write_shared,
                          __nv_bfloat16* x_perm, int num_sms, int* status, cudaStream_t st) {
  if (x_bf16 && !write_shared && T >= kGatherRowsMinTokens) {
    // rows of up to 96 KB of buffers per block: 6 warps at H = 4096
    const int row_bytes = H * 2;
    int wpb = (96 * 1024) / (2 * row_bytes);
    wpb = wpb < 1 ? 1 : (wpb > 8 ? 8 : wpb);
    const int want = (T + wpb - 1) / wpb;
    const int blocks = max(1, min(want, num_sms * 2));
    const size_t smem = static_cast<size_t>(wpb) * (2 * row_bytes + 16);
    return launch_pdl(gather_rows_kernel, dim3(blocks), dim3(32 * wpb), smem, st,
                      static_cast<const __nv_bfloat16*>(x), pos, T, k, H, x_perm, status);
  }
  const int nrows = rows_routed + (write_shared ? T : 0);
  const int want = (nrows + 7) / 8;
  const int blocks = max(1, min(want, num_sms * 8));
  if (x_bf16)
    return launch_pdl(gather_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, st,
                      static_cast<const __nv_bfloat16*>(x), perm, rows_routed, k, T, H,
                      write_shared ? 1 : 0, x_perm);
  return launch_pdl(gather_kernel<float>, dim3(blocks), dim3(256), 0, st,
                    static_cast<const float*>(x), perm, rows_routed, k, T, H, write_shared ? 1 : 0,
                    x_perm);
}

}  // namespace moe
