// The fused persistent MoE layer forward: K1-K7 in ONE launch.
//
// The pages' TPU design has a FusedEPMoE backend next to the grouped-matmul
// one (sglang-jax issue #1367 "Support Step 3.5 Flash", section "Reuse map",
// and sub-issue "FusedEPMoE performance backend switch"): routing, the expert
// FFNs and the combine in a single kernel.  This is its B200 counterpart for
// the CTA-pair regime (bf16 x and weights, from kPairMinTokens tokens): a
// persistent grid of 2-CTA clusters (one per two SMs, all co-resident) walks
// the phases of the layer, separated by grid-wide barriers:
//
//   R  router logits on the tensor cores: x . W1|W2|W3 (the three-term bf16
//      split of W_r; each term's K in two halves: six K parts, so the tiles
//      fill the pairs in even waves), pair MMAs of 256 expert rows x 256
//      tokens, fp32 partial logits, summed by the top-k          | barrier
//   K  top-k, one warp per token over the whole grid (the warp form of the
//      top-k kernels: boundary candidates recomputed in fp32)     | barrier
//   S  counting sort: chunk histograms | scan (one CTA) | stable scatter,
//      each separated by a barrier                                | barrier
//   G  the expert GEMMs as one tile list: every gate|up tile, then every down
//      tile.  A down tile waits (bounded) until all gate|up tiles of its
//      group's token block have stored their rows of h, through a per-block
//      readiness counter, instead of for the whole gate|up GEMM.     | barrier
//   C  combine: out[t] = sum_j y[pos(t, j)] + y[shared row t], fixed order.
//
// What the single launch removes: the launch boundaries between the nine
// kernels of the multi-launch path, the gather kernel and x_perm (the
// gate|up tiles of the routed experts read their token rows straight from x:
// two gather warps per CTA copy each row's 128-byte K chunks with cp.async
// into the 128B-swizzled operand slot), and the tail between the two GEMMs.
// y stays: the combine's fixed summation order (deterministic output) needs
// every contribution of a token.  Same tiles, same MMAs, same K order as the
// multi-launch path, so the outputs are bit-identical to it.
//
// Warps (256 threads per CTA): 0 TMA producer (weights, and token rows not
// gathered); 1 TMEM allocation, the MMA issuer (leader CTA) or, in the peer
// CTA, the forwarder of its gathered stages to the leader's full barrier;
// 2-5 epilogue; 6-7 token-row gather.  In the phases without MMAs all eight
// warps work.  Every wait is bounded (mbarriers, the grid barrier, the
// readiness counters): on expiry the CTA sets its abort flag and a device
// status bit and winds down.  No TMA multicast.
#include "combine_device.cuh"
#include "gemm_common.cuh"
#include "moe_internal.h"
#include "moe_ptx.cuh"
#include "pair_common.cuh"
#include "sort_device.cuh"
#include "topk_warp.cuh"

namespace moe {

namespace {

using namespace gemm;

constexpr int kFusedWarps = 8;
constexpr int kFusedThreads = 32 * kFusedWarps;
constexpr int kGatherWarp0 = 6;   // warps 6 and 7 gather token rows
constexpr int kGatherThreads = 64;
constexpr int kFusedGroups = kFusedMaxExperts + 1;

enum TileKind { kRt = 0, kGu = 1, kDn = 2 };

struct FusedShape : PairStage {
  static constexpr int BN = kPairBN;
  static constexpr int ACC_COLS = BN;                     // fp32 columns per accumulator buffer
  static constexpr int TMEM_COLS = 2 * ACC_COLS;
  static constexpr int BAR_BYTES = 256;
  static constexpr int STG_BYTES = kEpiRows * 32 * 2;     // one 16 x 32 bf16 output chunk
  static constexpr int XCH_BYTES = 2 * 8 * 32 * 4;        // gate|up exchange of one warp pair
  static constexpr int EPI_OFFSET = STAGES * STAGE_BYTES + BAR_BYTES;
  static constexpr int XCH_OFFSET = EPI_OFFSET + 4 * 2 * STG_BYTES;
  static constexpr int OKX_OFFSET = XCH_OFFSET + 2 * XCH_BYTES;
  static constexpr int WB_OFFSET = OKX_OFFSET + 64;       // down: per warp BN gate weights
  static constexpr int TAB_OFFSET = WB_OFFSET + 4 * BN * 4;
  // tiles_gu, tiles_dn, counts, row_start of up to kFusedGroups groups
  static constexpr int TAB_BYTES = 4 * (kFusedGroups + 1) * 4;
  static constexpr size_t SMEM = 1024 + static_cast<size_t>(TAB_OFFSET) + TAB_BYTES;
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
  static_assert(TMEM_COLS <= 512, "TMEM capacity");
  static_assert(1024 + STAGES * STAGE_BYTES + BAR_BYTES <= 256 * 1024, "descriptor range");
};

// Grid-wide barrier number `n` (0, 1, ...) on a counter that starts at zero:
// every CTA adds one and waits until all gridDim.x CTAs of barrier n have
// arrived.  Bounded: on expiry sets the abort flag and the status bit.
// Returns false when the CTA is aborting.
__device__ __forceinline__ bool grid_sync(unsigned int* counter, unsigned int n,
                                          volatile int* abort_flag, int* status,
                                          uint64_t limit_ns) {
  __syncthreads();
  if (threadIdx.x == 0 && !*abort_flag) {
    __threadfence();
    atomicAdd(counter, 1u);
    const unsigned int target = (n + 1u) * gridDim.x;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
      unsigned int v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
      if (v >= target) break;
      if (global_timer_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        atomicOr(status, kDevErrTimeout);
        break;
      }
      __nanosleep(64);
    }
  }
  __syncthreads();
  return !*abort_flag;
}

// Waits (bounded) until *counter >= target; then orders the caller's later
// TMA (async-proxy) reads of global memory after the writes it observed.
__device__ __forceinline__ bool wait_counter(const unsigned int* counter, unsigned int target,
                                             volatile int* abort_flag, int* status,
                                             uint64_t limit_ns) {
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
    if (v >= target) break;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicOr(status, kDevErrTimeout);
      return false;
    }
    __nanosleep(32);
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return true;
}

// mbar_wait with cluster-scope acquire: the leader's full barrier also
// counts the peer CTA's forwarded arrival (a cluster-scope release that
// covers the peer's gathered token rows).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity,
                                                  volatile int* abort, int* status,
                                                  uint64_t limit_ns) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait_cluster(bar, parity)) return true;
    if (*abort) return false;
    if (global_timer_ns() - t0 > limit_ns) {
      *abort = 1;
      atomicOr(status, kDevErrTimeout);
      return false;
    }
  }
}

// 16-byte global -> shared copy (cp.async, L2 only) and the arrival on an
// mbarrier of this CTA once every prior cp.async of the thread has landed
// (the barrier's count includes it: .noinc).
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src))
               : "memory");
}

__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Everything the fused forward reads and writes (device pointers).
struct FusedParams {
  const __nv_bfloat16* x;       // [T, H]
  __nv_bfloat16* out;           // [T, H]
  int T, H, E, k, I_pad;
  // router
  const float* bias;            // [E] or nullptr
  const float* router_t;        // [E, H] fp32 (candidate recomputation)
  float band;                   // guard band of the candidate recomputation
  int norm;
  float scale;
  int rt_mtiles;                // 256-row tiles of the packed router (rows past E_pad read 0)
  float* logits_out;            // optional [T, E]
  // workspace
  float* partial;               // [3][T][E]
  int* topk_idx;
  float* topk_w;
  uint32_t* masks;
  int* chunk_cnt;
  int* chunk_base;
  int* counts;                  // [G]
  int* row_start;               // [G + 1]
  int* tiles_gu;                // [G + 1]
  int* tiles_dn;                // [G + 1]
  int* perm;
  int* pos;
  float* w_perm;
  __nv_bfloat16* h;             // [T k + T, I_pad]
  __nv_bfloat16* y;             // [T k + T, H]
  unsigned int* sync;           // [0] grid barrier; [1 + b] readiness of token block b
  float limit, limit_shared;
  int* status;
  __nv_bfloat16* x_perm;        // non-null: the routed rows are gathered into x_perm in a
                                // phase of their own and read by TMA (else by the
                                // gather warps, straight from x)
  uint64_t wait_ns;             // limit of every bounded wait
  unsigned int ready_extra;     // self-check only: arrivals a down tile waits for beyond
                                // its token block's gate|up tiles (0 in a forward)
};

// One tile of the fused schedule, as every role decodes it.
struct FTile {
  int kind;
  int g, mt, nc, n_valid, nch;
  int z;          // router: K part (term of the split)
  bool gather;    // gate|up of a routed expert: token rows gathered from x
  int blk;        // gate|up / down: the token block's readiness counter
};

__device__ __forceinline__ FTile router_tile(const FusedParams& p, int w) {
  FTile t{};
  const int nb = (p.T + kPairBN - 1) / kPairBN;
  const int per_part = p.rt_mtiles * nb;
  t.kind = kRt;
  t.z = w / per_part;
  const int rem = w - t.z * per_part;
  t.nc = rem / p.rt_mtiles;
  t.mt = rem - t.nc * p.rt_mtiles;
  t.g = 0;
  t.nch = nb;
  t.n_valid = min(kPairBN, p.T - t.nc * kPairBN);
  return t;
}

__device__ __forceinline__ FTile gemm_tile(const GemmParams& gpu, const GemmParams& gpd, int n_gu,
                                           int w, int E, bool in_producer) {
  FTile t{};
  const bool gu = w < n_gu;
  const Tile d = gu ? decode_tile<kPairBN>(gpu, w) : decode_tile<kPairBN>(gpd, w - n_gu);
  t.kind = gu ? kGu : kDn;
  t.g = d.g;
  t.mt = d.mt;
  t.nc = d.nc;
  t.n_valid = d.n_valid;
  t.nch = d.nch;
  t.gather = in_producer && gu && d.g != E;
  t.blk = gpu.tile_start[d.g] / gpu.m_tiles + d.nc;
  return t;
}

// Tensor maps of the fused forward (K-block maps, see launch_gemm_gate_up_pair):
// weights of wide / narrow stages for the router, gate|up and down; token rows
// of x and of h with 128-row x 2 and 32-row x 3 K-block boxes; stores of h, y.
struct FusedMaps {
  CUtensorMap rt_w, rt_n, gu_w, gu_n, dn_w, dn_n, x_w, x_n, h_w, h_n, st_h, st_y, xp_w, xp_n;
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kFusedThreads, 1)
    moe_fused_kernel(const __grid_constant__ FusedMaps m, const FusedParams p) {
  using S = FusedShape;
  constexpr int BN = S::BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::STAGES * S::STAGE_BYTES);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * S::STAGES;
  const uint32_t gfull0 = empty0 + 8 * S::STAGES;
  const uint32_t tfull0 = gfull0 + 8 * S::STAGES;
  const uint32_t tempty0 = tfull0 + 16;
  const uint32_t drain = tempty0 + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * S::STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  static_assert((3 * S::STAGES + 5) * 8 + 8 <= S::BAR_BYTES, "barrier area");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  const int G = p.E + 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(full0 + 8 * s, 2);                 // leader: producer arming + (peer forward
                                                   // of gathered rows, or the producer again)
      mbar_init(empty0 + 8 * s, 1);                // one multicast commit
      mbar_init(gfull0 + 8 * s, kGatherThreads);   // this CTA's gather threads (gathered
                                                   // stages only)
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, 8);               // leader: 4 epilogue warps of each CTA
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    const CUtensorMap* maps[14] = {&m.rt_w, &m.rt_n, &m.gu_w, &m.gu_n, &m.dn_w,
                                   &m.dn_n, &m.x_w,  &m.x_n,  &m.h_w,  &m.h_n,
                                   &m.st_h, &m.st_y, &m.xp_w, &m.xp_n};
    for (int i = 0; i < (p.x_perm != nullptr ? 14 : 12); ++i) prefetch_tmap(maps[i]);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), S::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // role state carried from the router phase into the GEMM phase
  uint32_t it = 0;      // pipeline stages (producer, gather, forwarder, issuer)
  uint32_t tc = 0;      // accumulator buffers (issuer, epilogue)
  uint32_t chunks = 0;  // epilogue: staged output chunks (double buffer index)
  uint32_t gpar = 0;    // per slot: parity of its gather barrier (flips on gathered stages only)
  const uint32_t full_leader = mapa_shared(full0, 0);
  const uint32_t tempty_leader = mapa_shared(tempty0, 0);
  const uint64_t desc0 = sdesc_k_sw<128>(smem_u32(smem));

  // ------------------------------------------------------------------ roles
  // Every role walks the same tiles (w = pair, pair + n_pairs, ...) of a phase.
  auto run_tiles = [&](int phase, int n_tiles, const GemmParams& gpu, const GemmParams& gpd,
                       int n_gu) {
    auto tile_of = [&](int w) {
      return phase == 0 ? router_tile(p, w)
                        : gemm_tile(gpu, gpd, n_gu, w, p.E, p.x_perm == nullptr);
    };
    // router parts cover half of one bf16 term's K each (kFusedRouterParts)
    const int num_kb_of[3] = {p.H / 2 / kBK, p.H / kBK, p.I_pad / kBK};
    if (warp == 0) {
      // ---------------------------------------------------- TMA producer
      if (lane != 0) return;
      const uint64_t pol_first = l2_policy_evict_first();
      const uint64_t pol_normal = l2_policy_evict_normal();
      const uint64_t pol_b = l2_policy_evict_last();
      for (int w = pair; w < n_tiles; w += n_pairs) {
        if (*abort_flag) return;
        const FTile t = tile_of(w);
        const int half = ((t.n_valid + 15) & ~15) >> 1;
        const bool narrow = narrow_tile(t.n_valid);
        const int ks = narrow ? S::KS_N : S::KS_W;
        const int num_kb = num_kb_of[t.kind];
        const int n_st = (num_kb + ks - 1) / ks;
        const CUtensorMap* ma;
        const CUtensorMap* mb;
        int a_row, b_row, a_kb0 = 0, b_kb0 = 0;
        if (t.kind == kRt) {
          // part z: K blocks [z, z + 1) * H / 2 of the packed W1 | W2 | W3, against
          // x's first or second half of K
          ma = narrow ? &m.rt_n : &m.rt_w;
          mb = narrow ? &m.x_n : &m.x_w;
          a_row = t.mt * 2 * kBM + static_cast<int>(rank) * kBM;
          a_kb0 = t.z * (p.H / 2 / kBK);
          b_kb0 = (t.z & 1) * (p.H / 2 / kBK);
          b_row = t.nc * BN + static_cast<int>(rank) * half;
        } else if (t.kind == kGu) {
          ma = narrow ? &m.gu_n : &m.gu_w;
          a_row = t.g * 2 * p.I_pad + t.mt * 2 * kBM + static_cast<int>(rank) * 64;
          if (t.g == p.E) {  // the shared expert's rows are x itself
            mb = narrow ? &m.x_n : &m.x_w;
            b_row = t.nc * BN + static_cast<int>(rank) * half;
          } else {           // (x_perm: the gathered rows; unused when gathered here)
            mb = narrow ? &m.xp_n : &m.xp_w;
            b_row = gpu.row_start[t.g] + t.nc * BN + static_cast<int>(rank) * half;
          }
        } else {
          ma = narrow ? &m.dn_n : &m.dn_w;
          mb = narrow ? &m.h_n : &m.h_w;
          a_row = t.g * p.H + t.mt * 2 * kBM + static_cast<int>(rank) * kBM;
          b_row = gpu.row_start[t.g] + t.nc * BN + static_cast<int>(rank) * half;
          // h rows of this token block: every gate|up tile of it stored
          if (!wait_counter(p.sync + 1 + t.blk,
                            8u * static_cast<unsigned>(gpu.m_tiles) + p.ready_extra, abort_flag,
                            p.status, p.wait_ns))
            return;
        }
        const uint32_t a_bytes = narrow ? S::A_BYTES_N : S::A_BYTES_W;
        const uint32_t b_bytes = t.gather ? 0u : (narrow ? S::B_BYTES_N : S::B_BYTES_W);
        const uint32_t b_off = narrow ? S::B_OFF_N : S::B_OFF_W;
        const uint64_t pol_a = (t.kind == kRt || t.nch > 1) ? pol_normal : pol_first;
        for (int st = 0; st < n_st; ++st) {
          const uint32_t s = it % S::STAGES;
          const uint32_t ph = (it / S::STAGES) & 1u;
          if (!mbar_wait(empty0 + 8 * s, ph ^ 1u, abort_flag, p.status, p.wait_ns)) return;
          if (rank == 0) {
            mbar_arrive_expect_tx(full0 + 8 * s, 2 * (a_bytes + b_bytes));
            // a stage without gathered rows needs no forward from the peer:
            // its second arrival comes from here
            if (!t.gather) mbar_arrive(full0 + 8 * s);
          }
          const uint32_t fb = full_leader + 8 * s;
          const uint32_t sa = smem_u32(smem + s * S::STAGE_BYTES);
          const int kb0 = st * ks;
          if (t.kind == kGu)
            tma_load_4d_pair(sa, ma, fb, 0, a_row, 0, kb0, pol_a);
          else
            tma_load_3d_pair(sa, ma, fb, 0, a_row, a_kb0 + kb0, pol_a);
          if (!t.gather) tma_load_3d_pair(sa + b_off, mb, fb, 0, b_row, b_kb0 + kb0, pol_b);
          ++it;
        }
      }
    } else if (warp >= kGatherWarp0) {
      // ---------------------------------------------------- token-row gather
      // Thread g (0..63) of the two gather warps copies chunk c = g % 8 (16
      // bytes) of rows r = g / 8 + 8 j of this CTA's token half: per tile it
      // looks its rows' tokens up in perm once and keeps their source
      // pointers; per stage and K sub-block each copy is one cp.async to the
      // 128B-swizzled slot (chunk c of row r at (c ^ r % 8) * 16, and r % 8 =
      // g / 8 for every j).  Eight consecutive threads cover one row's 128
      // bytes.  Rows past the group are not copied: their MMA columns are
      // never stored.  The two warps never wait for each other.
      constexpr int kRowsPerThread = (kPairBN / 2) / 8;  // 16
      const int g = threadIdx.x - kGatherWarp0 * 32;
      const int c = g & 7, rg = g >> 3;
      const uint32_t swz = static_cast<uint32_t>((c ^ rg) << 4);
      const __nv_bfloat16* src[kRowsPerThread];
      for (int w = pair; w < n_tiles; w += n_pairs) {
        if (*abort_flag) return;
        const FTile t = tile_of(w);
        const int half = ((t.n_valid + 15) & ~15) >> 1;
        const bool narrow = narrow_tile(t.n_valid);
        const int ks = narrow ? S::KS_N : S::KS_W;
        const int num_kb = num_kb_of[t.kind];
        const int n_st = (num_kb + ks - 1) / ks;
        if (t.gather) {
          const int cnt = gpu.counts[t.g];
          const int* pg = p.perm + gpu.row_start[t.g];  // (written in this launch: plain loads)
          const int rbase = t.nc * BN + static_cast<int>(rank) * half;
#pragma unroll
          for (int j = 0; j < kRowsPerThread; ++j) {
            const int r = rg + 8 * j;
            src[j] = nullptr;
            if (r < half && rbase + r < cnt)
              src[j] = p.x + static_cast<size_t>(pg[rbase + r] / p.k) * p.H + c * 8;
          }
        }
        const uint32_t b_off = narrow ? S::B_OFF_N : S::B_OFF_W;
        const uint32_t sub_b = narrow ? S::SUB_BN : S::SUB_BW;
        if (!t.gather) {  // nothing to copy; keep the stage count
          it += n_st;
          continue;
        }
        for (int st = 0; st < n_st; ++st) {
          const uint32_t s = it % S::STAGES;
          const uint32_t ph = (it / S::STAGES) & 1u;
          int ok = 1;
          if (lane == 0)
            ok = mbar_wait(empty0 + 8 * s, ph ^ 1u, abort_flag, p.status, p.wait_ns) ? 1 : 0;
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) return;
          {
            const uint32_t sb = smem_u32(smem + s * S::STAGE_BYTES) + b_off + rg * 128 + swz;
            const int kb0 = st * ks;
            const int nsub = min(ks, num_kb - kb0);
            for (int hh = 0; hh < nsub; ++hh) {
              const uint32_t dh = sb + hh * sub_b;
              const int ko = (kb0 + hh) * kBK;
#pragma unroll
              for (int j = 0; j < kRowsPerThread; ++j)
                if (src[j] != nullptr) cp_async_16(dh + j * 8 * 128, src[j] + ko);
            }
            cp_async_arrive_noinc(gfull0 + 8 * s);
          }
          ++it;
        }
      }
    } else if (warp == 1) {
      if (rank != 0) {
        // ------------------------------------------ peer: forward its gathered stages
        if (lane != 0) return;
        for (int w = pair; w < n_tiles; w += n_pairs) {
          if (*abort_flag) return;
          const FTile t = tile_of(w);
          const bool narrow = narrow_tile(t.n_valid);
          const int ks = narrow ? S::KS_N : S::KS_W;
          const int n_st = (num_kb_of[t.kind] + ks - 1) / ks;
          if (!t.gather) {
            it += n_st;
            continue;
          }
          for (int st = 0; st < n_st; ++st) {
            const uint32_t s = it % S::STAGES;
            if (!mbar_wait(gfull0 + 8 * s, (gpar >> s) & 1u, abort_flag, p.status, p.wait_ns))
              return;
            gpar ^= 1u << s;
            fence_proxy_async_smem();  // the gathered rows, before the leader's MMAs read them
            mbar_arrive_cluster(full_leader + 8 * s);
            ++it;
          }
        }
        return;
      }
      // ---------------------------------------------- leader: MMA issuer
      if (lane != 0) return;
      for (int w = pair; w < n_tiles; w += n_pairs) {
        if (*abort_flag) return;
        const FTile t = tile_of(w);
        const int n_mma = (t.n_valid + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(2 * kBM, n_mma);
        const uint32_t buf = tc & 1u;
        const uint32_t tph = (tc >> 1) & 1u;
        if (!mbar_wait(tempty0 + 8 * buf, tph ^ 1u, abort_flag, p.status, p.wait_ns)) return;
        tc_fence_after();
        const uint32_t d = tmem_base + buf * S::ACC_COLS;
        const bool narrow = narrow_tile(t.n_valid);
        const int ks = narrow ? S::KS_N : S::KS_W;
        const int num_kb = num_kb_of[t.kind];
        const int n_st = (num_kb + ks - 1) / ks;
        const uint32_t b_off = narrow ? S::B_OFF_N : S::B_OFF_W;
        for (int st = 0; st < n_st; ++st) {
          const uint32_t s = it % S::STAGES;
          const uint32_t ph = (it / S::STAGES) & 1u;
          // (cluster-scope acquire only where the peer forwarded gathered rows)
          if (t.gather ? !mbar_wait_cluster(full0 + 8 * s, ph, abort_flag, p.status, p.wait_ns)
                       : !mbar_wait(full0 + 8 * s, ph, abort_flag, p.status, p.wait_ns))
            return;
          if (t.gather) {
            if (!mbar_wait(gfull0 + 8 * s, (gpar >> s) & 1u, abort_flag, p.status, p.wait_ns))
              return;
            gpar ^= 1u << s;
            fence_proxy_async_smem();
          }
          tc_fence_after();
          const uint64_t ad = desc0 + static_cast<uint64_t>((s * S::STAGE_BYTES) >> 4);
          const uint64_t bd = ad + static_cast<uint64_t>(b_off >> 4);
          const int nsub = min(ks, num_kb - st * ks);
          if (narrow)
            issue_stage_pair<S::KS_N, S::SUB_A, S::SUB_BN>(d, ad, bd, idesc, nsub, st == 0);
          else
            issue_stage_pair<S::KS_W, S::SUB_A, S::SUB_BW>(d, ad, bd, idesc, nsub, st == 0);
          tc_commit_pair_mc(empty0 + 8 * s, 3);  // frees the stage in both CTAs
          ++it;
        }
        tc_commit_pair_mc(tfull0 + 8 * buf, 3);  // accumulators ready in both CTAs
        ++tc;
      }
    } else {
      // ---------------------------------------------------- epilogue (warps 2-5)
      const int q = warp & 3;  // the TMEM lane quadrant this warp may read
      const int ew = warp - 2;
      uint8_t* stg_base = smem + S::EPI_OFFSET + ew * 2 * S::STG_BYTES;
      float* wbuf = reinterpret_cast<float*>(smem + S::WB_OFFSET) + ew * BN;
      for (int w = pair; w < n_tiles; w += n_pairs) {
        const FTile t = tile_of(w);
        const uint32_t buf = tc & 1u;
        const uint32_t tph = (tc >> 1) & 1u;
        const size_t row0 =
            t.kind == kRt ? 0 : static_cast<size_t>(gpu.row_start[t.g]) + static_cast<size_t>(t.nc) * BN;
        float wl[BN / 32];
        if (t.kind == kDn) {
#pragma unroll
          for (int mm = 0; mm < BN / 32; ++mm)
            wl[mm] = lane + 32 * mm < t.n_valid ? p.w_perm[row0 + lane + 32 * mm] : 0.f;
        }
        int ok = 1;
        if (lane == 0) ok = mbar_wait(tfull0 + 8 * buf, tph, abort_flag, p.status, p.wait_ns) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (t.kind == kGu) {
          // the two warps of a gate|up pair meet at named barriers, so they
          // continue or stop together
          volatile int* okx = reinterpret_cast<volatile int*>(smem + S::OKX_OFFSET) +
                              (q & 1) * 4 + (tc & 1u) * 2;
          if (lane == 0) okx[q < 2 ? 0 : 1] = ok;
          named_bar_sync(1 + (q & 1), 64);
          ok = okx[0] & okx[1];
        }
        if (!ok) return;
        tc_fence_after();
        const uint32_t taddr =
            tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * S::ACC_COLS;
        if (t.kind == kRt) {
          // fp32 partial logits: lane = expert mt*256 + 128 r + 32 q + lane
          const int e = t.mt * 2 * kBM + static_cast<int>(rank) * kBM + q * 32 + lane;
          float* dst = p.partial + (static_cast<size_t>(t.z) * p.T + t.nc * BN) * p.E + e;
          for (int c0 = 0; c0 < t.n_valid; c0 += kEpiRows) {
            uint32_t ra[16];
            tmem_ld_x16(taddr + c0, ra);
            tmem_ld_wait();
            if (e < p.E) {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (c0 + i < t.n_valid)
                  dst[static_cast<size_t>(c0 + i) * p.E] = __uint_as_float(ra[i]);
            }
          }
        } else if (t.kind == kGu) {
          // lanes 0-63 gate, 64-127 up of features [mt*128 + 64 r, +64): warp q
          // (gate, q < 2) and warp q + 2 (up) share features fbase + lane; the
          // gate warp finishes tokens 0-7 of each 16-token chunk, the up warp
          // tokens 8-15
          const bool is_gate = q < 2;
          const int pr = q & 1;
          const uint32_t bar_id = 1 + pr;
          float* xch = reinterpret_cast<float*>(smem + S::XCH_OFFSET + pr * S::XCH_BYTES);
          const int fbase = t.mt * kBM + static_cast<int>(rank) * 64 + pr * 32;
          __nv_bfloat16* outp = p.h + row0 * p.I_pad + fbase + lane;
          const float L = (t.g == p.E) ? p.limit_shared : p.limit;
          for (int c0 = 0; c0 < t.n_valid; c0 += kEpiRows) {
            uint32_t ra[16];
            tmem_ld_x16(taddr + c0, ra);
            tmem_ld_wait();
            const bool full = c0 + kEpiRows <= t.n_valid;
            const uint32_t buf_off = (chunks & 1u) * S::STG_BYTES;
            if (full && is_gate && chunks >= 2 && lane == 0) bulk_wait_group_read<1>();
#pragma unroll
            for (int i = 0; i < 8; ++i)
              xch[(is_gate ? 0 : 256) + i * 32 + lane] = __uint_as_float(ra[is_gate ? 8 + i : i]);
            named_bar_sync(bar_id, 64);
            float hv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              float a = is_gate ? __uint_as_float(ra[i]) : xch[i * 32 + lane];
              float u = is_gate ? xch[256 + i * 32 + lane] : __uint_as_float(ra[8 + i]);
              if (L > 0.f) {
                a = fminf(a, L);
                u = fminf(fmaxf(u, -L), L);
              }
              hv[i] = a / (1.0f + __expf(-a)) * u;
            }
            const int r0 = is_gate ? 0 : 8;
            if (full) {
              __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(
                  smem + S::EPI_OFFSET + (pr * 2) * 2 * S::STG_BYTES + buf_off);
#pragma unroll
              for (int i = 0; i < 8; ++i) stg[(r0 + i) * 32 + lane] = __float2bfloat16_rn(hv[i]);
              fence_proxy_async_smem();
            } else {
#pragma unroll
              for (int i = 0; i < 8; ++i)
                if (c0 + r0 + i < t.n_valid)
                  outp[static_cast<size_t>(c0 + r0 + i) * p.I_pad] = __float2bfloat16_rn(hv[i]);
            }
            named_bar_sync(bar_id, 64);
            if (full) {
              if (is_gate && lane == 0) {
                const uint32_t src = smem_u32(smem + S::EPI_OFFSET +
                                              (pr * 2) * 2 * S::STG_BYTES + buf_off);
                tma_store_2d(&m.st_h, src, fbase, static_cast<int>(row0) + c0);
                bulk_commit_group();
              }
              ++chunks;
            }
          }
        } else {
          const int feat = t.mt * 2 * kBM + static_cast<int>(rank) * kBM + q * 32 + lane;
          __nv_bfloat16* outp = p.y + row0 * p.H + feat;
#pragma unroll
          for (int mm = 0; mm < BN / 32; ++mm) wbuf[lane + 32 * mm] = wl[mm];
          __syncwarp();
          for (int c0 = 0; c0 < t.n_valid; c0 += kEpiRows) {
            uint32_t ra[16];
            tmem_ld_x16(taddr + c0, ra);
            float wv[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) wv[i] = wbuf[c0 + i];
            tmem_ld_wait();
            if (c0 + kEpiRows <= t.n_valid) {
              const uint32_t buf_off = (chunks & 1u) * S::STG_BYTES;
              if (chunks >= 2 && lane == 0) bulk_wait_group_read<1>();
              __syncwarp();
              __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(stg_base + buf_off);
#pragma unroll
              for (int i = 0; i < kEpiRows; ++i)
                stg[i * 32 + lane] = __float2bfloat16_rn(__uint_as_float(ra[i]) * wv[i]);
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(&m.st_y, smem_u32(stg), feat - lane, static_cast<int>(row0) + c0);
                bulk_commit_group();
              }
              ++chunks;
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (c0 + i < t.n_valid)
                  outp[static_cast<size_t>(c0 + i) * p.H] =
                      __float2bfloat16_rn(__uint_as_float(ra[i]) * wv[i]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty_leader + 8 * buf);
        if (t.kind == kGu) {
          // this warp's rows of h for the tile are written: count them for the
          // down tiles of the block (8 warps of the pair per gate|up tile)
          if (lane == 0) {
            bulk_wait_group_all();
            fence_proxy_async_global();
          }
          __syncwarp();
          __threadfence();
          if (lane == 0) atomicAdd(p.sync + 1 + t.blk, 1u);
        }
        ++tc;
      }
      if (lane == 0) {
        bulk_wait_group_all();  // h / y fully written
        fence_proxy_async_global();
      }
    }
  };

  GemmParams none{};
  unsigned int nbar = 0;
  float* scratch = reinterpret_cast<float*>(smem);  // the operand ring, between GEMM phases

  // ------------------------------------------------------------ R: router
  {
    const int nb = (p.T + kPairBN - 1) / kPairBN;
    run_tiles(0, kFusedRouterParts * p.rt_mtiles * nb, none, none, 0);
  }
  if (!grid_sync(p.sync, nbar++, abort_flag, p.status, p.wait_ns)) goto teardown;

  // ------------------------------------------------------------ K: top-k
  {
    float* s_bias = scratch;
    int* c_lists = reinterpret_cast<int*>(scratch + p.E);
    for (int e = threadIdx.x; e < p.E; e += blockDim.x)
      s_bias[e] = p.bias != nullptr ? p.bias[e] : 0.f;
    __syncthreads();
    TopkRefine rf{};
    rf.x = p.x;
    rf.w_t = p.router_t;
    rf.H = p.H;
    rf.band = p.band;
    const int gw = blockIdx.x * kFusedWarps + warp;
    for (int t = gw; t < p.T; t += gridDim.x * kFusedWarps)
      topk::topk_warp_token<kFusedMPL>(t, p.partial, kFusedRouterParts, p.T, p.E, p.k, s_bias,
                                       c_lists + warp * 32, p.norm, p.scale, p.topk_idx,
                                       p.topk_w, p.logits_out, rf);
  }
  if (!grid_sync(p.sync, nbar++, abort_flag, p.status, p.wait_ns)) goto teardown;

  // ------------------------------------------------------------ S: counting sort
  {
    const int nch = (p.T + kSortChunk - 1) / kSortChunk;
    uint32_t* sm = reinterpret_cast<uint32_t*>(scratch);
    for (int c = blockIdx.x; c < nch; c += gridDim.x) {
      sort::hist_chunk(c, p.topk_idx, p.T, p.k, p.E, p.masks, p.chunk_cnt, sm);
      __syncthreads();
    }
    if (!grid_sync(p.sync, nbar++, abort_flag, p.status, p.wait_ns)) goto teardown;
    if (blockIdx.x == 0)
      sort::scan_block(p.chunk_cnt, nch, p.T, p.k, p.E, p.T, kPairBN, kPairBN, p.I_pad / kBM,
                       p.H / (2 * kBM), p.chunk_base, p.counts, p.row_start, p.tiles_gu,
                       p.tiles_dn, reinterpret_cast<int*>(scratch));
    if (!grid_sync(p.sync, nbar++, abort_flag, p.status, p.wait_ns)) goto teardown;
    for (int c = blockIdx.x; c < nch; c += gridDim.x) {
      sort::scatter_chunk(c, p.topk_idx, p.topk_w, p.T, p.k, p.E, p.masks, p.chunk_base,
                          p.row_start, p.perm, p.pos, p.w_perm, sm);
      __syncthreads();
    }
  }
  if (!grid_sync(p.sync, nbar++, abort_flag, p.status, p.wait_ns)) goto teardown;

  // ------------------------------------------------------------ gather phase
  if (p.x_perm != nullptr) {
    // x_perm[r] = x[perm[r] / k], one warp per row at a time over the grid
    const int rows = p.T * p.k;
    const int nvec = p.H / 8;
    for (int r = blockIdx.x * kFusedWarps + warp; r < rows; r += gridDim.x * kFusedWarps) {
      const int t = p.perm[r] / p.k;
      const uint4* src = reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(t) * p.H);
      uint4* dst = reinterpret_cast<uint4*>(p.x_perm + static_cast<size_t>(r) * p.H);
      for (int v = lane; v < nvec; v += 32) dst[v] = src[v];
    }
    __threadfence();
    fence_proxy_async_global();  // before the GEMM phase's TMA reads of x_perm
    if (!grid_sync(p.sync, nbar++, abort_flag, p.status, p.wait_ns)) goto teardown;
  }

  // ------------------------------------------------------------ G: expert GEMMs
  {
    // group tables in shared memory: tiles_gu, tiles_dn, counts, row_start
    int* tab = reinterpret_cast<int*>(smem + S::TAB_OFFSET);
    for (int i = threadIdx.x; i <= G; i += blockDim.x) {
      tab[i] = p.tiles_gu[i];
      tab[(kFusedGroups + 1) + i] = p.tiles_dn[i];
      tab[3 * (kFusedGroups + 1) + i] = p.row_start[i];
      if (i < G) tab[2 * (kFusedGroups + 1) + i] = p.counts[i];
    }
    __syncthreads();
    GemmParams gpu{}, gpd{};
    gpu.G = gpd.G = G;
    gpu.E = gpd.E = p.E;
    gpu.counts = gpd.counts = tab + 2 * (kFusedGroups + 1);
    gpu.row_start = gpd.row_start = tab + 3 * (kFusedGroups + 1);
    gpu.tile_start = tab;
    gpd.tile_start = tab + (kFusedGroups + 1);
    gpu.m_tiles = p.I_pad / kBM;
    gpd.m_tiles = p.H / (2 * kBM);
    const int n_gu = gpu.tile_start[G];
    const int n_dn = gpd.tile_start[G];
    run_tiles(1, n_gu + n_dn, gpu, gpd, n_gu);
  }
  if (!grid_sync(p.sync, nbar++, abort_flag, p.status, p.wait_ns)) goto teardown;

  // ------------------------------------------------------------ C: combine
  {
    // one (token, 8-element vector) item per thread at a time, over the whole
    // grid (many independent row loads in flight); the same fixed order as
    // the combine kernel: j = 0..k-1, then the shared row
    const int nvec = p.H / 8;
    const size_t items = static_cast<size_t>(p.T) * nvec;
    for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < items;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
      const int t = static_cast<int>(i / nvec);
      const int v = static_cast<int>(i - static_cast<size_t>(t) * nvec);
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      const int* pt = p.pos + static_cast<size_t>(t) * p.k;
      const size_t shared_row = static_cast<size_t>(p.T) * p.k + t;
      if (p.k == 8) {  // the layer's top-8: all nine rows in flight at once
        uint4 q[9];
#pragma unroll
        for (int j = 0; j < 9; ++j)
          q[j] = *reinterpret_cast<const uint4*>(
              p.y + (j < 8 ? static_cast<size_t>(pt[j]) : shared_row) * p.H + v * 8);
#pragma unroll
        for (int j = 0; j < 9; ++j) combine::add8(acc, q[j]);
      } else {
        for (int j = 0; j < p.k; ++j)
          combine::add8(acc, p.y + static_cast<size_t>(pt[j]) * p.H + v * 8);
        combine::add8(acc, p.y + shared_row * p.H + v * 8);
      }
      combine::store8(p.out + static_cast<size_t>(t) * p.H + v * 8, acc);
    }
  }

teardown:
  // in-flight work this CTA started: the leader sees every armed stage land,
  // the gather threads' copies complete, the issuer's MMAs complete
  if (warp == 0 && lane == 0 && rank == 0) {
    const uint32_t used = it < static_cast<uint32_t>(S::STAGES) ? it : S::STAGES;
    for (uint32_t s = 0; s < used; ++s) {
      const uint32_t last = (it - 1u) - ((it - 1u - s) % S::STAGES);
      mbar_wait(full0 + 8 * s, (last / S::STAGES) & 1u, nullptr, p.status, p.wait_ns);
    }
  }
  if (warp >= kGatherWarp0) cp_async_wait_all();
  if (warp == 1 && lane == 0 && rank == 0 && it > 0) {
    tc_commit_pair(drain);
    mbar_wait(drain, 0, nullptr, p.status, p.wait_ns);
  }
  tc_fence_before();
  __syncthreads();
  // neither CTA leaves (nor frees TMEM) while its peer may still use its
  // shared memory, barriers or TMEM
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, S::TMEM_COLS);
  }
}

int g_fused_grid = 0;  // CTAs per launch: twice the co-resident clusters

}  // namespace

size_t fused_smem_bytes() { return FusedShape::SMEM; }

cudaError_t fused_configure_device(int num_sms) {
  cudaError_t e = cudaFuncSetAttribute(moe_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(FusedShape::SMEM));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms & ~1), 1, 1);
  cfg.blockDim = dim3(kFusedThreads, 1, 1);
  cfg.dynamicSmemBytes = FusedShape::SMEM;
  cudaLaunchAttribute attr{};
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if ((e = cudaOccupancyMaxActiveClusters(&clusters, moe_fused_kernel, &cfg)) != cudaSuccess)
    return e;
  g_fused_grid = 2 * (clusters < num_sms / 2 ? clusters : num_sms / 2);
  return g_fused_grid > 0 ? cudaSuccess : cudaErrorInvalidConfiguration;
}

int fused_grid() { return g_fused_grid; }

cudaError_t launch_fused(const FusedLaunch& f, cudaStream_t st) {
  if (g_fused_grid <= 0) return cudaErrorInvalidConfiguration;
  FusedMaps m{};
  m.rt_w = f.rt_w;
  m.rt_n = f.rt_n;
  m.gu_w = f.gu_w;
  m.gu_n = f.gu_n;
  m.dn_w = f.dn_w;
  m.dn_n = f.dn_n;
  m.x_w = f.x_w;
  m.x_n = f.x_n;
  m.h_w = f.h_w;
  m.h_n = f.h_n;
  m.st_h = f.st_h;
  m.st_y = f.st_y;
  m.xp_w = f.xp_w;
  m.xp_n = f.xp_n;
  FusedParams p{};
  p.x = f.x;
  p.out = f.out;
  p.T = f.T;
  p.H = f.H;
  p.E = f.E;
  p.k = f.k;
  p.I_pad = f.I_pad;
  p.bias = f.bias;
  p.router_t = f.router_t;
  p.band = f.band;
  p.norm = f.norm;
  p.scale = f.scale;
  p.rt_mtiles = f.rt_mtiles;
  p.logits_out = f.logits_out;
  p.partial = f.partial;
  p.topk_idx = f.topk_idx;
  p.topk_w = f.topk_w;
  p.masks = f.masks;
  p.chunk_cnt = f.chunk_cnt;
  p.chunk_base = f.chunk_base;
  p.counts = f.counts;
  p.row_start = f.row_start;
  p.tiles_gu = f.tiles_gu;
  p.tiles_dn = f.tiles_dn;
  p.perm = f.perm;
  p.pos = f.pos;
  p.w_perm = f.w_perm;
  p.h = f.h;
  p.y = f.y;
  p.sync = f.sync;
  p.limit = f.limit;
  p.limit_shared = f.limit_shared;
  p.status = f.status;
  p.x_perm = f.x_perm;
  p.wait_ns = f.wait_ns > 0 ? f.wait_ns : kWaitLimitNs;
  p.ready_extra = f.ready_extra;
  // (not a programmatic-dependent launch: the first phase reads x at once)
  moe_fused_kernel<<<g_fused_grid, kFusedThreads, FusedShape::SMEM, st>>>(m, p);
  return cudaGetLastError();
}

}  // namespace moe
