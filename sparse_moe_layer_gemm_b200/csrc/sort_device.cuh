// Device code of the deterministic token-to-expert grouping (K3), shared by
// the sort kernels (permute.cu) and the fused persistent MoE kernel
// (fused_moe.cu).  Definition kept: perm lists the pair ids t * k + j of
// expert 0, then expert 1, ..., each in ascending t; pos[t * k + j] is the
// pair's slot in perm; the shared expert is group E with the T identity rows
// [T*k, T*k + T).  No order-dependent atomics: a chunk of kSortChunk tokens
// records, per expert, a 128-bit mask of its tokens that chose that expert
// (atomicOr gives the same mask in any order), and a pair's rank inside its
// chunk is the popcount of the mask bits below its token.
//
// Every function here is called by all threads of a block (it uses
// threadIdx.x / blockDim.x strides and __syncthreads).
#pragma once

#include "moe_internal.h"

namespace moe {
namespace sort {

constexpr int kMaskWords = kSortChunk / 32;  // 4

// Histogram of chunk c: its masks (masks[c][E][4]) and per-expert counts
// (chunk_cnt[c][E]); sm: E * kMaskWords words of shared memory.
__device__ __forceinline__ void hist_chunk(int c, const int* __restrict__ topk_idx, int T, int k,
                                           int E, uint32_t* __restrict__ masks,
                                           int* __restrict__ chunk_cnt, uint32_t* sm) {
  const int t0 = c * kSortChunk;
  const int nt = min(kSortChunk, T - t0);
  for (int i = threadIdx.x; i < E * kMaskWords; i += blockDim.x) sm[i] = 0u;
  __syncthreads();
  for (int p = threadIdx.x; p < nt * k; p += blockDim.x) {
    const int tl = p / k;
    const int e = topk_idx[static_cast<size_t>(t0) * k + p];
    if (static_cast<unsigned>(e) < static_cast<unsigned>(E))
      atomicOr(&sm[e * kMaskWords + (tl >> 5)], 1u << (tl & 31));
  }
  __syncthreads();
  uint32_t* mo = masks + static_cast<size_t>(c) * E * kMaskWords;
  for (int i = threadIdx.x; i < E * kMaskWords; i += blockDim.x) mo[i] = sm[i];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int n = 0;
#pragma unroll
    for (int q = 0; q < kMaskWords; ++q) n += __popc(sm[e * kMaskWords + q]);
    chunk_cnt[static_cast<size_t>(c) * E + e] = n;
  }
}

// Warp-wide exclusive prefix over the G = E + 1 groups of the row counts and
// of the GEMM tile counts (ceil(rows / bn) token tiles x m_tiles weight
// tiles, with each GEMM's own bn).  Called by one full warp; cnt_s holds
// the G row counts; the last group (the shared expert) starts at row
// shared_row0 (T*k: equal to the prefix unless a shard dropped pairs).  When
// start_s is given, the row starts are also left there for the caller.
__device__ __forceinline__ void scan_groups(const int* cnt_s, int G, int bn_gu, int bn_dn, int mt_gu, int mt_dn,
                            int shared_row0, int* __restrict__ counts,
                            int* __restrict__ row_start, int* __restrict__ tiles_gu,
                            int* __restrict__ tiles_dn, int* start_s) {
  const int lane = threadIdx.x & 31;
  const int per = (G + 31) / 32;
  const int g0 = min(G, lane * per), g1 = min(G, g0 + per);
  int s_rows = 0, s_gu = 0, s_dn = 0;
  for (int g = g0; g < g1; ++g) {
    const int n = cnt_s[g];
    s_rows += n;
    s_gu += (n + bn_gu - 1) / bn_gu * mt_gu;
    s_dn += (n + bn_dn - 1) / bn_dn * mt_dn;
  }
  int i_rows = s_rows, i_gu = s_gu, i_dn = s_dn;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, i_rows, off);
    const int b = __shfl_up_sync(0xffffffffu, i_gu, off);
    const int d = __shfl_up_sync(0xffffffffu, i_dn, off);
    if (lane >= off) {
      i_rows += a;
      i_gu += b;
      i_dn += d;
    }
  }
  int b_rows = i_rows - s_rows, b_gu = i_gu - s_gu, b_dn = i_dn - s_dn;
  for (int g = g0; g < g1; ++g) {
    const int n = cnt_s[g];
    counts[g] = n;
    row_start[g] = g == G - 1 ? shared_row0 : b_rows;
    if (start_s != nullptr) start_s[g] = row_start[g];
    tiles_gu[g] = b_gu;
    tiles_dn[g] = b_dn;
    b_rows += n;
    b_gu += (n + bn_gu - 1) / bn_gu * mt_gu;
    b_dn += (n + bn_dn - 1) / bn_dn * mt_dn;
  }
  if (lane == 31) {
    row_start[G] = shared_row0 + cnt_s[G - 1];
    tiles_gu[G] = i_gu;
    tiles_dn[G] = i_dn;
  }
}

// Per expert: running offsets of the chunks (chunk_base); then warp 0 forms
// the prefixes over the groups.  cnt_s: E + 1 ints of shared memory.
__device__ __forceinline__ void scan_block(const int* __restrict__ chunk_cnt, int nch, int T,
                                           int k, int E, int shared_rows, int bn_gu, int bn_dn,
                                           int mt_gu, int mt_dn, int* __restrict__ chunk_base,
                                           int* __restrict__ counts, int* __restrict__ row_start,
                                           int* __restrict__ tiles_gu, int* __restrict__ tiles_dn,
                                           int* cnt_s) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int c = 0; c < nch; ++c) {
      chunk_base[static_cast<size_t>(c) * E + e] = run;
      run += chunk_cnt[static_cast<size_t>(c) * E + e];
    }
    cnt_s[e] = run;
  }
  if (threadIdx.x == 0) cnt_s[E] = shared_rows;
  __syncthreads();
  if (threadIdx.x < 32)
    scan_groups(cnt_s, E + 1, bn_gu, bn_dn, mt_gu, mt_dn, T * k, counts, row_start, tiles_gu,
                tiles_dn, nullptr);
}

// Rank of token tl among the tokens of this chunk that chose the expert whose
// 128-bit mask is m: the number of mask bits below tl.
__device__ __forceinline__ int chunk_rank(const uint32_t* m, int tl) {
  const int wd = tl >> 5;
  int rank = __popc(m[wd] & ((1u << (tl & 31)) - 1u));
  for (int q = 0; q < wd; ++q) rank += __popc(m[q]);
  return rank;
}

// Stable scatter of chunk c: perm, pos and the rows' gate weights w_perm
// (1 for the shared rows of the chunk's tokens); sm: E * kMaskWords words.
__device__ __forceinline__ void scatter_chunk(int c, const int* __restrict__ topk_idx,
                                              const float* __restrict__ topk_w, int T, int k,
                                              int E, const uint32_t* __restrict__ masks,
                                              const int* __restrict__ chunk_base,
                                              const int* __restrict__ row_start,
                                              int* __restrict__ perm, int* __restrict__ pos,
                                              float* __restrict__ w_perm, uint32_t* sm) {
  const int t0 = c * kSortChunk;
  const int nt = min(kSortChunk, T - t0);
  const uint32_t* mi = masks + static_cast<size_t>(c) * E * kMaskWords;
  for (int i = threadIdx.x; i < E * kMaskWords; i += blockDim.x) sm[i] = mi[i];
  __syncthreads();
  for (int p = threadIdx.x; p < nt * k; p += blockDim.x) {
    const int tl = p / k;
    const size_t pair = static_cast<size_t>(t0) * k + p;
    const int e = topk_idx[pair];
    if (static_cast<unsigned>(e) >= static_cast<unsigned>(E)) {  // another shard's expert
      pos[pair] = -1;
      continue;
    }
    const int slot = row_start[e] + chunk_base[static_cast<size_t>(c) * E + e] +
                     chunk_rank(sm + e * kMaskWords, tl);
    perm[slot] = static_cast<int>(pair);
    pos[pair] = slot;
    w_perm[slot] = topk_w[pair];
  }
  const int shared0 = T * k;
  for (int tl = threadIdx.x; tl < nt; tl += blockDim.x) w_perm[shared0 + t0 + tl] = 1.0f;
}

}  // namespace sort
}  // namespace moe
