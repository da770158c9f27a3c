// The dense SwiGLU MLP at decode-sized T (at most kSkMaxTokens tokens) in ONE
// persistent launch: stream-K over both GEMMs in 2 kSkGroups passes,
// synchronised by data flow.  With one group (the setting; more groups were
// measured slower):
//
//   A  gate|up                                    fp32 partials per segment
//      reduced per h tile once its segments are stored:
//      h = silu(min(a, L)) * clip(u, -L, L), bf16
//   B  down, each K block's h rows loaded once they exist (the down weights
//      stream as soon as a CTA's ring is free of gate|up stages)
//      then out = the down partials summed, bf16 or fp32
//
// (sglang-jax issue #1367 "Support Step 3.5 Flash", section "Model
// configuration", MLP bullet: the first three layers are dense, intermediate
// 11264; llm-atlas "Step-3.5-Flash", "Raw config fields".)
//
// Why stream-K: at T <= 128 one token block covers every token, so a GEMM
// has only I_pad / 128 (gate|up, 256 packed rows each) or H / 256 (down)
// weight tiles -- 88 and 16 at the model's sizes, fewer than the 148 SMs.
// A pass's work is the list of its (tile, 64-deep K block) units, tile-major;
// CTA c takes the contiguous units [c U / G, (c + 1) U / G), so every SM
// streams the same number of weight bytes (+-1 K block).  A CTA's range is
// cut at tile boundaries into segments; each segment's raw fp32 accumulators
// go to a slot of their own.  Every CTA reduces an equal share of a pass's
// output rows (tile j, token t) from L2, summing the segments in CTA order
// (fixed by the grid size: deterministic, and independent of T and of the
// batch).
//
// Passes: the down GEMM needs h, and h needs every gate|up segment.  With
// gate|up split into groups of h tiles, a group's reduction could run while
// the SM streams the next group, and a down pass would need only its group's
// h; but the extra segment boundaries cost more partials than the overlap
// gains, so the kernel runs one group (two passes).  Under full HBM load
// every global round trip -- a counter, a fence, an L2 load -- takes
// microseconds, so the reductions never run on the warps that drain the
// accumulators.
//
// No grid barrier: counters in device memory owned by the layer carry the
// dependencies -- per tile of each pass the stored segments (one count per
// store warp and segment), per h tile the reduced rows.  They are never
// reset: a forward's targets are the running totals (forward count x
// segments, and the sum of T over the layer's forwards), so no launch-time
// clearing breaks the programmatic launch chain, and the forwards of one
// layer must run on the device in the order they were issued.  The totals
// live on the device too: each forward reads them after its pdl_wait and
// the last CTA to finish advances them, so a launch captured in a CUDA graph
// computes the right targets at every replay.
//
// Warps (480 threads): 0 TMA producer; 1, 2 tcgen05.mma issuers (one 128-row
// accumulator each: gate and up, or two 128-row blocks of H); 3-6 store
// warps (TMEM -> fp32 slots, one per lane quadrant); 7-14 reducers of h; at
// the end every warp reduces the output rows.  Every wait is bounded; on expiry the CTA sets its abort flag and the device
// status bit and winds down.  No TMA multicast.
#include "dense_streamk.h"
#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {

namespace {

constexpr int kSkEpiWarp0 = 3;
constexpr int kSkEpiWarps = 4;                     // store warps, one per TMEM lane quadrant
constexpr int kSkRedWarp0 = kSkEpiWarp0 + kSkEpiWarps;
constexpr int kSkRedWarps = 8;                     // reducers
constexpr int kSkWarps = kSkRedWarp0 + kSkRedWarps;
constexpr int kSkBatchH = 6;    // h rows: segments whose (gate, up) loads are in flight together
constexpr int kSkBatchOut = 16; // output rows: segments whose loads are in flight together
constexpr int kSkThreads = 32 * kSkWarps;
constexpr int kSkTileRows = 2 * kBM;               // weight rows per tile (two accumulators)
constexpr int kSkABytes = kSkTileRows * kBK * 2;   // 32 KB of weights per stage
constexpr int kSkRingBytes = 200 * 1024;           // operand ring
constexpr int kSkMaxStages = 6;
constexpr int kSkBarBytes = 256;
constexpr size_t kSkSmem = 1024 + kSkRingBytes + kSkBarBytes;
static_assert(kSkSmem <= 227 * 1024, "shared memory per CTA");
static_assert(1024 + kSkRingBytes <= 256 * 1024, "descriptor range");

struct SkParams {
  int T, n_mma;          // tokens; the MMA's N (T rounded up to 16)
  int H, I_pad;
  int stages, stage_bytes;
  SkPass pass[kSkPasses];
  int max_seg[kSkPasses];         // segment slots per CTA
  float* parts[kSkPasses];        // [grid][max_seg][T][256] fp32
  unsigned int* seg_cnt[kSkPasses];  // per tile of the pass: stored segments x epilogue warps
  unsigned int* h_cnt;            // per h tile: reduced rows
  unsigned int* epoch;            // [3]: forwards completed on this path, the sum of their
                                  // T, CTAs done with the current forward
  float limit;                    // SwiGLU clamp (<= 0: none)
  __nv_bfloat16* h;               // [T, I_pad]
  void* out;                      // [T, H]
  int out_f32;
  int* status;
  uint64_t wait_ns;
};

// Unit arithmetic is 32-bit: a pass has U = tiles x K blocks <= 65536 units
// (I_pad <= 32768, H <= 16384) and U x grid < 2^32.  CTA c's units start at
// floor(c U / G) (a table in shared memory, one entry per CTA and pass).

// The CTA whose range holds unit u: the largest c with floor(c U / G) <= u.
__device__ __forceinline__ uint32_t unit_owner(uint32_t u, uint32_t U, uint32_t G) {
  const uint32_t c = ((u + 1) * G - 1) / U;
  return c < G - 1 ? c : G - 1;
}

struct Seg {
  int tile, kb0, nkb, ord;
};

// Walks the units [lo, hi) of one pass as segments (one per tile touched).
struct SegWalk {
  uint32_t u, hi, nkb;
  int ord;
  __device__ SegWalk(uint32_t lo, uint32_t hi_, uint32_t nkb_) : u(lo), hi(hi_), nkb(nkb_), ord(0) {}
  __device__ bool next(Seg& s) {
    if (u >= hi) return false;
    const uint32_t tile = u / nkb;
    const uint32_t kb0 = u - tile * nkb;
    const uint32_t n = hi - u < nkb - kb0 ? hi - u : nkb - kb0;
    s.tile = static_cast<int>(tile);
    s.kb0 = static_cast<int>(kb0);
    s.nkb = static_cast<int>(n);
    s.ord = ord++;
    u += n;
    return true;
  }
};

// Waits (bounded) until a running counter reaches target (wrap-safe); with
// `proxy`, then orders this thread's later TMA reads after what the counted
// writers stored.
__device__ __forceinline__ bool wait_count(const unsigned int* cnt, unsigned int target,
                                           volatile int* abort_flag, int* status,
                                           uint64_t limit_ns, bool proxy) {
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
    if (static_cast<int>(v - target) >= 0) break;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicOr(status, kDevErrTimeout);
      return false;
    }
    __nanosleep(32);
  }
  if (proxy) fence_proxy_async_global();
  return true;
}

// Publishes a warp's global stores (all lanes, ordered by the warp barrier)
// with one release increment of a counter (no round trip for the warp);
// `proxy`: the stores are read next by TMA.
__device__ __forceinline__ void warp_publish(unsigned int* cnt, unsigned int add, int lane,
                                             bool proxy) {
  if (proxy) fence_proxy_async_global();
  __syncwarp();
  if (lane == 0 && add > 0)
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(cnt), "r"(add) : "memory");
}

__device__ __forceinline__ float silu_mul(float a, float u, float L) {
  if (L > 0.f) {
    a = fminf(a, L);
    u = fminf(fmaxf(u, -L), L);
  }
  return a / (1.0f + __expf(-a)) * u;
}

__device__ __forceinline__ void add4(float4& a, const float4& b) {
  a.x += b.x;
  a.y += b.y;
  a.z += b.z;
  a.w += b.w;
}

__device__ __forceinline__ uint2 pack_bf16x4(float a, float b, float c, float d) {
  const __nv_bfloat162 lo2 = __floats2bfloat162_rn(a, b);
  const __nv_bfloat162 hi2 = __floats2bfloat162_rn(c, d);
  uint2 v;
  v.x = *reinterpret_cast<const uint32_t*>(&lo2);
  v.y = *reinterpret_cast<const uint32_t*>(&hi2);
  return v;
}

// The segments of tile j in one pass: CTAs cf .. cl (those with units), in
// CTA order.
struct TileSegs {
  int cf, cl, nseg;
};

__device__ __forceinline__ TileSegs tile_segs(int j, uint32_t nkb, uint32_t U, uint32_t G,
                                              const uint32_t* lo, int lane) {
  TileSegs ts;
  ts.cf = static_cast<int>(unit_owner(j * nkb, U, G));
  ts.cl = static_cast<int>(unit_owner((j + 1) * nkb - 1, U, G));
  ts.nseg = 0;
  for (int base = ts.cf; base <= ts.cl; base += 32) {
    const int cs = base + lane;
    ts.nseg += __popc(__ballot_sync(0xffffffffu, cs <= ts.cl && lo[cs + 1] > lo[cs]));
  }
  return ts;
}

// Adds, in segment order, token t's partial rows of tile j (one pass) to
// acc: lane l reads columns col0 + 4 l .. + 3 and, with NH = 2, the same
// columns + 128.  Up to BATCH segments' loads are in flight together, then
// added in order.  The slots were published before (wait_count) and
// are read from L2 (ld.global.cg: never a line cached in L1 by an earlier
// forward).
template <int NH, int BATCH>
__device__ __forceinline__ void sum_segments(const float* parts, int max_seg, int T, int t, int j,
                                             const TileSegs& ts, uint32_t nkb, const uint32_t* lo,
                                             int lane, int col0, float4 (&acc)[NH]) {
  for (int base = ts.cf; base <= ts.cl; base += 32) {
    const int cs = base + lane;
    const bool has = cs <= ts.cl && lo[cs + 1] > lo[cs];
    // this lane's segment: slot (cs, ord), token row t
    const int ord = has ? j - static_cast<int>(lo[cs] / nkb) : 0;
    const int my_off = has ? ((cs * max_seg + ord) * T + t) * kSkTileRows : 0;
    unsigned m = __ballot_sync(0xffffffffu, has);
    while (m != 0u) {
      int off[BATCH];
      bool v[BATCH];
#pragma unroll
      for (int k = 0; k < BATCH; ++k) {
        v[k] = m != 0u;
        const int src = v[k] ? __ffs(m) - 1 : 0;
        if (v[k]) m &= m - 1u;
        off[k] = __shfl_sync(0xffffffffu, my_off, src);
      }
      float4 a[BATCH][NH];
#pragma unroll
      for (int k = 0; k < BATCH; ++k)
#pragma unroll
        for (int h = 0; h < NH; ++h)
          if (v[k])
            a[k][h] = __ldcg(reinterpret_cast<const float4*>(parts + off[k] + col0 + h * kBM +
                                                             4 * lane));
#pragma unroll
      for (int k = 0; k < BATCH; ++k)
#pragma unroll
        for (int h = 0; h < NH; ++h)
          if (v[k]) add4(acc[h], a[k][h]);
    }
  }
}

__global__ void __launch_bounds__(kSkThreads, 1)
    dense_streamk_kernel(const __grid_constant__ CUtensorMap tm_gu,
                         const __grid_constant__ CUtensorMap tm_dn,
                         const __grid_constant__ CUtensorMap tm_x,
                         const __grid_constant__ CUtensorMap tm_h, const SkParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kSkRingBytes);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * kSkMaxStages;
  const uint32_t tfull0 = empty0 + 8 * kSkMaxStages;
  const uint32_t tempty0 = tfull0 + 16;
  const uint32_t drain = tempty0 + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kSkMaxStages + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  static_assert((2 * kSkMaxStages + 5) * 8 + 8 <= kSkBarBytes, "barrier area");
  __shared__ uint32_t s_lo[kSkPasses][kSkMaxGrid + 1];  // first unit of each CTA, per pass
  __shared__ unsigned int s_target[2];                   // this forward's counter targets

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int c = blockIdx.x;
  const int n_mma = p.n_mma;
  const uint32_t acc_cols = 2 * n_mma;                     // one buffer: two accumulators
  const uint32_t tmem_cols = 4 * n_mma <= 256 ? 256u : 512u;

  for (int i = threadIdx.x; i <= G; i += blockDim.x)
#pragma unroll
    for (int q = 0; q < kSkPasses; ++q)
      s_lo[q][i] = static_cast<uint32_t>(i) * static_cast<uint32_t>(p.pass[q].tiles * p.pass[q].nkb) /
                   static_cast<uint32_t>(G);
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 2);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 2);
      mbar_init(tempty0 + 8 * b, kSkEpiWarps);
    }
    mbar_init(drain, 2);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_gu);
    prefetch_tmap(&tm_dn);
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_h);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish();
  }
  pdl_wait();  // x and the layer's counters come from the previous kernels of the stream
  if (threadIdx.x == 0) {
    // the counters' targets: the running totals of the forwards before this
    // one (written by the last CTA of the previous forward, whose grid has
    // completed), plus this one
    s_target[0] = __ldcg(p.epoch) + 1u;
    s_target[1] = __ldcg(p.epoch + 1) + static_cast<unsigned int>(p.T);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const unsigned int fwd = s_target[0];     // forwards on this path, this one included
  const unsigned int h_rows = s_target[1];  // the sum of their T (mod 2^32)
  const uint32_t b_bytes = static_cast<uint32_t>(n_mma) * 128u;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();   // weights: read once
      const uint64_t pol_b = l2_policy_evict_last();    // x and h: every tile reads them
      uint32_t it = 0;
      bool ok = true;
      int h_ready = -1;  // the last h tile seen complete
      for (int q = 0; q < kSkPasses && ok; ++q) {
        const SkPass ps = p.pass[q];
        const CUtensorMap* ma = ps.gemm == 0 ? &tm_gu : &tm_dn;
        const CUtensorMap* mb = ps.gemm == 0 ? &tm_x : &tm_h;
        SegWalk sw(s_lo[q][c], s_lo[q][c + 1], ps.nkb);
        Seg s;
        while (ok && sw.next(s)) {
          const int a_row = (ps.tile0 + s.tile) * kSkTileRows;
          for (int kb = ps.kb0 + s.kb0; kb < ps.kb0 + s.kb0 + s.nkb; ++kb) {
            const uint32_t st = it % p.stages;
            const uint32_t ph_it = (it / p.stages) & 1u;
            if (!mbar_wait(empty0 + 8 * st, ph_it ^ 1u, abort_flag, p.status, p.wait_ns)) {
              ok = false;
              break;
            }
            const uint32_t fb = full0 + 8 * st;
            mbar_arrive_expect_tx(fb, kSkABytes + b_bytes);
            const uint32_t sa = smem_u32(smem + st * p.stage_bytes);
            tma_load_2d(sa, ma, fb, kb * kBK, a_row, pol_w);
            tma_load_2d(sa + kBM * 128, ma, fb, kb * kBK, a_row + kBM, pol_w);
            // down: the K block's h rows (h tile kb / 2) once every row of
            // that tile is stored; on an abort the (unused) rows are loaded
            // anyway, so the stage completes and the teardown's wait ends
            if (ps.gemm == 1 && (kb >> 1) != h_ready) {
              if (ok && wait_count(p.h_cnt + (kb >> 1), h_rows, abort_flag, p.status,
                                   p.wait_ns, true))
                h_ready = kb >> 1;
              else
                ok = false;
            }
            tma_load_2d(sa + kSkABytes, mb, fb, kb * kBK, 0, pol_b);
            ++it;
            if (!ok) break;
          }
        }
      }
      // every armed stage must have landed before the CTA may exit
      const uint32_t used = it < static_cast<uint32_t>(p.stages) ? it : p.stages;
      for (uint32_t s = 0; s < used; ++s) {
        const uint32_t last = (it - 1u) - ((it - 1u - s) % p.stages);
        mbar_wait(full0 + 8 * s, (last / p.stages) & 1u, nullptr, p.status, p.wait_ns);
      }
    }
  } else if (warp <= 2) {
    // ------------------------------------------------------------ MMA issuers
    if (lane == 0) {
      const int me = warp - 1;  // accumulator: gate (or rows 0-127), up (or rows 128-255)
      const uint64_t desc0 = sdesc_k_sw<128>(smem_u32(smem));
      const uint32_t idesc = idesc_bf16_f32(kBM, n_mma);
      uint32_t it = 0, tc = 0;
      bool ok = true;
      for (int q = 0; q < kSkPasses && ok; ++q) {
        SegWalk sw(s_lo[q][c], s_lo[q][c + 1], p.pass[q].nkb);
        Seg s;
        while (ok && sw.next(s)) {
          const uint32_t buf = tc & 1u;
          const uint32_t tph = (tc >> 1) & 1u;
          if (!mbar_wait(tempty0 + 8 * buf, tph ^ 1u, abort_flag, p.status, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + buf * acc_cols + me * n_mma;
          for (int kb = 0; kb < s.nkb; ++kb) {
            const uint32_t st = it % p.stages;
            const uint32_t ph_it = (it / p.stages) & 1u;
            if (!mbar_wait(full0 + 8 * st, ph_it, abort_flag, p.status, p.wait_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t off = st * p.stage_bytes;
            const uint64_t ad = desc0 + static_cast<uint64_t>((off + me * kBM * 128) >> 4);
            const uint64_t bd = desc0 + static_cast<uint64_t>((off + kSkABytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
              tc_mma_bf16(d, ad + static_cast<uint64_t>((kk * 32) >> 4),
                          bd + static_cast<uint64_t>((kk * 32) >> 4), idesc,
                          (kb | kk) != 0 ? 1u : 0u);
            tc_commit(empty0 + 8 * st);  // frees the stage once these MMAs have read it
            ++it;
          }
          if (!ok) break;
          tc_commit(tfull0 + 8 * buf);
          ++tc;
        }
      }
      if (it > 0) {  // no MMA may still be writing TMEM at deallocation
        tc_commit(drain);
        mbar_wait(drain, 0, nullptr, p.status, p.wait_ns);
      }
    }
  } else if (warp < kSkRedWarp0) {
    // ------------------------------------------------------------ store warps
    // every segment: raw accumulators to its slot, published by each warp
    // once its 32 rows (both accumulators) are stored
    const int quad = warp & 3;  // the TMEM lane quadrant this warp may read
    uint32_t tc = 0;
    bool alive = true;
    for (int q = 0; q < kSkPasses && alive; ++q) {
      const size_t slot_floats = static_cast<size_t>(p.T) * kSkTileRows;
      SegWalk sw(s_lo[q][c], s_lo[q][c + 1], p.pass[q].nkb);
      Seg s;
      while (alive && sw.next(s)) {
        const uint32_t buf = tc & 1u;
        const uint32_t tph = (tc >> 1) & 1u;
        int ok = 1;
        if (lane == 0) ok = mbar_wait(tfull0 + 8 * buf, tph, abort_flag, p.status, p.wait_ns);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) {
          alive = false;
          break;
        }
        tc_fence_after();
        float* slot = p.parts[q] + static_cast<size_t>(c * p.max_seg[q] + s.ord) * slot_floats;
        for (int a = 0; a < 2; ++a) {
          const int row = a * kBM + quad * 32 + lane;
          const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                 buf * acc_cols + a * n_mma;
          for (int c0 = 0; c0 < p.T; c0 += 16) {
            uint32_t r[16];
            tmem_ld_x16(taddr + c0, r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (c0 + i < p.T) slot[static_cast<size_t>(c0 + i) * kSkTileRows + row] =
                  __uint_as_float(r[i]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty0 + 8 * buf);
        warp_publish(p.seg_cnt[q] + s.tile, 1u, lane, false);
        ++tc;
      }
    }
  } else {
    // ------------------------------------------------------------ reducers
    // An equal share of each gate|up pass's h rows (tile j, token t), one row
    // per warp at a time, once the tile's segments are stored.
    const int rw = warp - kSkRedWarp0;
    bool alive = true;
    for (int q = 0; q < kSkGroups && alive; ++q) {
      const SkPass ps = p.pass[q];
      const uint32_t R = static_cast<uint32_t>(ps.tiles * p.T);
      const uint32_t row_lo = static_cast<uint32_t>(c) * R / static_cast<uint32_t>(G);
      const uint32_t row_hi = static_cast<uint32_t>(c + 1) * R / static_cast<uint32_t>(G);
      int cur = -1;             // the tile whose segments are known complete
      unsigned int stored = 0;  // h rows of tile `cur` this warp has stored
      TileSegs ts{};
      for (uint32_t row = row_lo + rw; row < row_hi; row += kSkRedWarps) {
        const int j = static_cast<int>(row / p.T);
        const int t = static_cast<int>(row) - j * p.T;
        if (j != cur) {
          if (stored > 0) warp_publish(p.h_cnt + ps.tile0 + cur, stored, lane, true);
          stored = 0;
          ts = tile_segs(j, ps.nkb, ps.tiles * ps.nkb, G, s_lo[q], lane);
          int ok = 1;
          if (lane == 0)
            ok = wait_count(p.seg_cnt[q] + j, kSkEpiWarps * ts.nseg * fwd, abort_flag,
                            p.status, p.wait_ns, false);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          __syncwarp();  // the other lanes' loads after lane 0's acquire
          if (!ok) {
            alive = false;
            break;
          }
          cur = j;
        }
        // h[t][jh * 128 + 4 lane ..]: gate columns 4 lane.., up 128 + 4 lane..
        float4 acc[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
        sum_segments<2, kSkBatchH>(p.parts[q], p.max_seg[q], p.T, t, j, ts, ps.nkb, s_lo[q], lane, 0, acc);
        const float L = p.limit;
        *reinterpret_cast<uint2*>(p.h + static_cast<size_t>(t) * p.I_pad +
                                  (ps.tile0 + j) * kBM + 4 * lane) =
            pack_bf16x4(silu_mul(acc[0].x, acc[1].x, L), silu_mul(acc[0].y, acc[1].y, L),
                        silu_mul(acc[0].z, acc[1].z, L), silu_mul(acc[0].w, acc[1].w, L));
        ++stored;
      }
      if (stored > 0) warp_publish(p.h_cnt + ps.tile0 + cur, stored, lane, true);
    }
  }

  __syncwarp();  // the producer's and issuers' warps reconverge
  {
    // ------------------------------------------------ the output, every warp
    // An equal share of the output rows, each as two column halves, one per
    // warp at a time, summing the down passes' segments in pass order.
    bool alive = !*abort_flag;
    if (alive) {
      // out[t][j * 256 + half * 128 + 4 lane ..]
      const int tb = p.pass[kSkGroups].tiles;
      const uint32_t R = static_cast<uint32_t>(tb * p.T);
      const uint32_t row_lo = static_cast<uint32_t>(c) * R / static_cast<uint32_t>(G);
      const uint32_t row_hi = static_cast<uint32_t>(c + 1) * R / static_cast<uint32_t>(G);
      int cur = -1;
      for (uint32_t item = warp; item < 2 * (row_hi - row_lo) && alive; item += kSkWarps) {
        const uint32_t row = row_lo + (item >> 1);
        const int half = static_cast<int>(item & 1u);
        const int j = static_cast<int>(row / p.T);
        const int t = static_cast<int>(row) - j * p.T;
        if (j != cur) {  // every down pass's segments of tile j stored
          int ok = 1;
          for (int q = kSkGroups; q < kSkPasses && ok; ++q) {
            const SkPass ps = p.pass[q];
            if (ps.nkb == 0) continue;
            const TileSegs ts = tile_segs(j, ps.nkb, ps.tiles * ps.nkb, G, s_lo[q], lane);
            if (lane == 0)
              ok = wait_count(p.seg_cnt[q] + j, kSkEpiWarps * ts.nseg * fwd, abort_flag,
                              p.status, p.wait_ns, false);
            ok = __shfl_sync(0xffffffffu, ok, 0);
          }
          __syncwarp();  // the other lanes' loads after lane 0's acquires
          if (!ok) {
            alive = false;
            break;
          }
          cur = j;
        }
        float4 acc[1] = {make_float4(0.f, 0.f, 0.f, 0.f)};
        for (int q = kSkGroups; q < kSkPasses; ++q) {
          const SkPass ps = p.pass[q];
          if (ps.nkb == 0) continue;
          const TileSegs ts = tile_segs(j, ps.nkb, ps.tiles * ps.nkb, G, s_lo[q], lane);
          sum_segments<1, kSkBatchOut>(p.parts[q], p.max_seg[q], p.T, t, j, ts, ps.nkb, s_lo[q], lane,
                          half * kBM, acc);
        }
        const size_t o = static_cast<size_t>(t) * p.H + j * kSkTileRows + half * kBM + 4 * lane;
        if (p.out_f32)
          *reinterpret_cast<float4*>(static_cast<float*>(p.out) + o) = acc[0];
        else
          *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.out) + o) =
              pack_bf16x4(acc[0].x, acc[0].y, acc[0].z, acc[0].w);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    // the last CTA to finish moves the running totals on for the next
    // forward (which reads them after its pdl_wait, once this grid is done)
    __threadfence();
    if (atomicAdd(p.epoch + 2, 1u) == static_cast<unsigned int>(G) - 1u) {
      p.epoch[0] = fwd;
      p.epoch[1] = h_rows;
      p.epoch[2] = 0u;
      __threadfence();
    }
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

int g_sk_grid = 0;

}  // namespace

int dense_streamk_max_seg(int tiles, int nkb, int grid) {
  const long long U = static_cast<long long>(tiles) * nkb;
  int best = 0;
  for (int c = 0; c < grid && U > 0; ++c) {
    const long long lo = static_cast<long long>(c) * U / grid;
    const long long hi = static_cast<long long>(c + 1) * U / grid;
    if (hi <= lo) continue;
    const int n = static_cast<int>((hi - 1) / nkb - lo / nkb) + 1;
    if (n > best) best = n;
  }
  return best;
}

cudaError_t dense_streamk_configure_device(int num_sms) {
  cudaError_t e = cudaFuncSetAttribute(dense_streamk_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSkSmem));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dense_streamk_kernel, kSkThreads,
                                                    kSkSmem);
  if (e != cudaSuccess) return e;
  // one CTA per SM, all co-resident (CTAs wait on one another's counters)
  g_sk_grid = per_sm >= 1 ? num_sms : 0;
  return g_sk_grid > 0 ? cudaSuccess : cudaErrorInvalidConfiguration;
}

int dense_streamk_grid() { return g_sk_grid; }

cudaError_t launch_dense_streamk(const DenseStreamK& d, cudaStream_t st) {
  if (g_sk_grid <= 0 || d.T < 1 || d.T > kSkMaxTokens) return cudaErrorInvalidConfiguration;
  SkParams p{};
  p.T = d.T;
  p.n_mma = (d.T + 15) & ~15;
  p.H = d.H;
  p.I_pad = d.I_pad;
  p.stage_bytes = kSkABytes + p.n_mma * 128;
  p.stages = kSkRingBytes / p.stage_bytes;
  if (p.stages > kSkMaxStages) p.stages = kSkMaxStages;
  dense_streamk_passes(d.H, d.I_pad, p.pass);
  unsigned int* cnt = d.counters;
  for (int q = 0; q < kSkPasses; ++q) {
    p.max_seg[q] = d.max_seg[q];
    p.parts[q] = d.parts[q];
    p.seg_cnt[q] = cnt;
    cnt += p.pass[q].tiles;
  }
  p.h_cnt = cnt;
  p.epoch = cnt + d.I_pad / kBM;  // after the h tiles' counts (one per 128 features of h)
  p.limit = d.limit;
  p.h = d.h;
  p.out = d.out;
  p.out_f32 = d.out_f32 ? 1 : 0;
  p.status = d.status;
  p.wait_ns = kWaitLimitNs;
  return launch_pdl(dense_streamk_kernel, dim3(g_sk_grid), dim3(kSkThreads), kSkSmem, st, d.tm_gu,
                    d.tm_dn, d.tm_x, d.tm_h, p);
}

}  // namespace moe
