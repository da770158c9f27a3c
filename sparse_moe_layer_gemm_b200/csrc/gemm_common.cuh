// Device-side pieces shared by the expert-GEMM kernels (one CTA per tile and
// CTA pairs): the tile decode of the grouped problem, the group tables in
// shared memory and the output chunk size of the epilogues.
#pragma once

#include "moe_internal.h"

namespace moe {
namespace gemm {

// Rows per output chunk of the epilogues (one tcgen05.ld x16; one TMA store
// of 16 rows x 32 features).
constexpr int kEpiRows = 16;

// Shared-memory bytes of the group tables (tile_start, counts, row_start).
constexpr int kTabBytes = (3 * kMaxGroups + 1) * 4;

struct Tile {
  int g, mt, nc, n_valid, nch;  // nch: token blocks of the group
  int kz;                       // K part (single_rows with k_parts > 1), else 0
};

// Token blocks per ordering chunk (see decode_tile).
constexpr int kChunk = 4;

// Tile w -> (group, weight tile, token block).  tile_start is the exclusive
// prefix of per-group tile counts, so the group is the last g with
// tile_start[g] <= w (empty groups are skipped naturally).  Within a group
// the tiles run in chunks of kChunk token blocks; inside a chunk weight-tile
// major, token-block minor.  Consecutive tiles go to different CTAs at about
// the same time, so the (up to kChunk) readers of a weight tile share one
// pass through L2, while a chunk's token rows (kChunk x 128 rows) stay in L2
// across its weight tiles; an expert's weights (21 MB gate|up, 10.5 MB down)
// stay in L2 from one chunk to the next.
template <int BN>
__device__ __forceinline__ Tile decode_tile(const GemmParams& p, int w) {
  int g, local, rows, kz = 0;
  if (p.single_rows > 0) {
    g = 0;
    rows = p.single_rows;
    const int per_part = p.m_tiles * ((rows + BN - 1) / BN);
    kz = w / per_part;
    local = w - kz * per_part;
  } else {
    int lo = 0, hi = p.G;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.tile_start[mid] <= w)
        lo = mid;
      else
        hi = mid;
    }
    g = lo;
    local = w - p.tile_start[lo];
    rows = p.counts[lo];
  }
  Tile t;
  t.g = g;
  t.kz = kz;
  t.nch = (rows + BN - 1) / BN;
  const int per_chunk = p.m_tiles * kChunk;
  const int cc = local / per_chunk;
  const int rem = local - cc * per_chunk;
  const int in_chunk = min(kChunk, t.nch - cc * kChunk);  // token blocks in this chunk
  t.mt = rem / in_chunk;
  t.nc = cc * kChunk + (rem - t.mt * in_chunk);
  t.n_valid = min(BN, rows - t.nc * BN);
  return t;
}

template <int BN>
__device__ __forceinline__ int total_tiles(const GemmParams& p) {
  if (p.single_rows > 0)
    return (p.k_parts > 1 ? p.k_parts : 1) * p.m_tiles * ((p.single_rows + BN - 1) / BN);
  return p.tile_start[p.G];
}

__device__ __forceinline__ int group_row0(const GemmParams& p, int g) {
  return p.single_rows > 0 ? 0 : p.row_start[g];
}

// Copies the group tables into shared memory (all threads of the CTA; visible
// after the next __syncthreads) and returns parameters that read them there.
// Every role decodes every tile; from shared memory that is a short search
// instead of a chain of dependent global loads, which take microseconds each
// while the weights stream through L2.
__device__ __forceinline__ GemmParams stage_group_tables(const GemmParams& p, int* tab) {
  GemmParams gp = p;
  if (p.single_rows > 0) return gp;
  for (int i = threadIdx.x; i <= p.G; i += blockDim.x) tab[i] = p.tile_start[i];
  for (int i = threadIdx.x; i < p.G; i += blockDim.x) {
    tab[kMaxGroups + 1 + i] = p.counts[i];
    tab[2 * kMaxGroups + 1 + i] = p.row_start[i];
  }
  gp.tile_start = tab;
  gp.counts = tab + kMaxGroups + 1;
  gp.row_start = gp.counts + kMaxGroups;
  return gp;
}

}  // namespace gemm
}  // namespace moe
