// K5 / K6 for large token counts: the same grouped gate|up and down GEMMs as
// grouped_gemm.cu, computed by pairs of CTAs with the 2-SM UMMA
// (tcgen05.mma.cta_group::2, M = 256).
//
// Why: the issue cost of one tcgen05.mma is ~60 (one SM) to ~100 (SM pair)
// cycles whatever its size, and one accumulator chain needs ~110-170 cycles
// per step, so 128-row x <=128-token MMAs leave the tensor cores idle much of
// the time once a tile has enough tokens to be compute-bound.  A pair MMA of
// 256 weight rows x 256 tokens keeps both SMs' tensor cores busy from a
// single issuing thread and a single accumulator chain (128 cycles of work
// per SM per instruction), with each SM's accumulator (128 rows x 256
// columns fp32) small enough to double-buffer in TMEM; and a 256-token tile
// reads each weight tile half as often as a 128-token one.
//
// Operand split of the pair MMA: CTA r supplies weight rows [128 r, 128 r +
// 128) of the tile and tokens [r N/2, (r + 1) N/2), and holds accumulator rows
// [128 r, 128 r + 128) x all N tokens in its TMEM.
//   gate|up: a tile is 128 features of one expert; CTA r loads the gate and the
//            up rows of features [64 r, 64 r + 64) (one 4-D box), so its
//            accumulator holds gate in lanes 0-63 and up in lanes 64-127 for
//            the same features; the epilogue pairs warp q (gate) with warp
//            q + 2 (up) through shared memory for the SwiGLU.
//   down:    a tile is 256 features; CTA r loads features [128 r, 128 r + 128).
//
// Pipeline stages (3 slots of 64 KB per CTA) carry several 64-deep K
// sub-blocks of both operands, each operand brought by ONE TMA load per stage
// (a 4-D box for the gate|up weights, 3-D boxes whose last dimension walks the
// K sub-blocks otherwise).  The weight stream is latency-bound at prefill
// sizes: a slot's round trip is the load's latency plus the issue of its
// MMAs, and only three slots fit.  So a tile whose token half is at most 32
// rows (most experts' tiles at prefill) uses a narrow stage: 3 K sub-blocks
// of weights (48 KB) and 3 of 32 token rows (12 KB), where a wide tile's
// stage holds 2 sub-blocks of weights and 2 of 128 token rows: 50 % more
// weight bytes in flight for the same ring.
//
// Roles per CTA (6 warps): warp 0 TMA producer (both CTAs: own halves, every
// load completing on the leader's full barrier); warp 1 TMEM allocation (both)
// and MMA issue (leader CTA only, one thread); warps 2-5 epilogue (both).
// Stage release and accumulator-ready signals are tcgen05.commit multicasts to
// both CTAs; accumulator release is one arrival per epilogue warp of both
// CTAs on the leader's barrier.  Every wait is bounded (moe_ptx.cuh).  No TMA
// multicast.
#include "gemm_common.cuh"
#include "moe_internal.h"
#include "moe_ptx.cuh"
#include "pair_common.cuh"

namespace moe {

namespace {

using namespace gemm;

template <int MODE>
struct PairShape : PairStage {
  static constexpr bool GU = MODE == kModeGateUp;
  static constexpr int BN = kPairBN;
  static constexpr int THREADS = 32 * 6;
  static constexpr int ACC_COLS = BN;                    // fp32 columns per accumulator buffer
  static constexpr int TMEM_COLS = 2 * ACC_COLS;
  static constexpr int BAR_BYTES = 256;
  static constexpr int STG_BYTES = kEpiRows * 32 * 2;    // one 16 x 32 bf16 output chunk
  static constexpr int XCH_BYTES = 2 * 8 * 32 * 4;       // gate|up exchange of one warp pair
  static constexpr int EPI_OFFSET = STAGES * STAGE_BYTES + BAR_BYTES;
  static constexpr int OKX_OFFSET = EPI_OFFSET + 4 * 2 * STG_BYTES + 2 * XCH_BYTES;
  static constexpr int WB_OFFSET = EPI_OFFSET + 4 * 2 * STG_BYTES;  // down: per warp BN gate weights
  static constexpr int EPI_BYTES = 4 * 2 * STG_BYTES + (GU ? 2 * XCH_BYTES + 64 : 4 * BN * 4);
  static constexpr int TAB_OFFSET = EPI_OFFSET + EPI_BYTES;
  static constexpr size_t SMEM = 1024 + static_cast<size_t>(TAB_OFFSET) + kTabBytes;
  static_assert((2 * STAGES + 5) * 8 + 8 <= BAR_BYTES, "barrier area");
  static_assert(1024 + STAGES * STAGE_BYTES + BAR_BYTES <= 256 * 1024, "descriptor range");
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
  static_assert(TMEM_COLS <= 512, "TMEM capacity");
};

// tmAw / tmAn: the weights of a wide / narrow stage (gate|up: 4-D boxes of
// 64 gate + 64 up rows x 2 or 3 K sub-blocks; down: 3-D boxes of 128 rows x 2
// or 3 K sub-blocks).  tmBw / tmBshw (128 rows x 2 K sub-blocks) and tmB /
// tmBsh (32 rows x 3 K sub-blocks): token rows (x_perm or h; tmBsh / tmBshw
// the shared expert's rows of x, gate|up only).  tmOut: h or y with
// 32-feature x 16-row boxes.  p.num_kb is K / 64 (K sub-blocks).
template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairShape<MODE>::THREADS, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmAw,
                             const __grid_constant__ CUtensorMap tmAn,
                             const __grid_constant__ CUtensorMap tmB,
                             const __grid_constant__ CUtensorMap tmBsh,
                             const __grid_constant__ CUtensorMap tmBw,
                             const __grid_constant__ CUtensorMap tmBshw,
                             const __grid_constant__ CUtensorMap tmOut, const GemmParams p) {
  using S = PairShape<MODE>;
  constexpr bool GU = S::GU;
  constexpr int BN = S::BN;
  extern __shared__ uint8_t smem_raw[];
  // same dynamic shared-memory base in both CTAs, so the leader's operand
  // descriptors address the same offsets in its peer
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::STAGES * S::STAGE_BYTES);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * S::STAGES;
  const uint32_t tfull0 = empty0 + 8 * S::STAGES;
  const uint32_t tempty0 = tfull0 + 16;
  const uint32_t drain = tempty0 + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S::STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);   // leader: its producer's expect-tx arrival
      mbar_init(empty0 + 8 * s, 1);  // one multicast commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);   // one multicast commit
      mbar_init(tempty0 + 8 * b, 8);  // leader: 4 epilogue warps of each CTA
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmAw);
    prefetch_tmap(&tmAn);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmBw);
    if (GU) {
      prefetch_tmap(&tmBsh);
      prefetch_tmap(&tmBshw);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), S::TMEM_COLS);
    tmem_relinquish_pair();
  }
  // everything above touched only this pair's resources; from here on the
  // previous kernel's outputs are read
  pdl_wait();
  const GemmParams gp = stage_group_tables(p, reinterpret_cast<int*>(smem + S::TAB_OFFSET));
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = total_tiles<BN>(gp);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_first = l2_policy_evict_first();
      const uint64_t pol_normal = l2_policy_evict_normal();
      const uint64_t pol_b = l2_policy_evict_last();
      const uint32_t full_leader = mapa_shared(full0, 0);
      uint32_t it = 0;
      for (int w = pair; w < total; w += n_pairs) {
        if (*abort_flag) break;
        const Tile t = decode_tile<BN>(gp, w);
        const int half = ((t.n_valid + 15) & ~15) >> 1;  // this CTA's token rows of the MMA
        const bool narrow = narrow_tile(t.n_valid);
        const int ks = narrow ? S::KS_N : S::KS_W;
        const int n_st = (p.num_kb + ks - 1) / ks;
        const bool sh = GU && t.g == p.E;
        const CUtensorMap* mb = narrow ? (sh ? &tmBsh : &tmB) : (sh ? &tmBshw : &tmBw);
        const CUtensorMap* ma = narrow ? &tmAn : &tmAw;
        const int b_row = (sh ? p.shared_b_row0 : group_row0(gp, t.g)) + t.nc * BN +
                          static_cast<int>(rank) * half;
        // gate|up: rows of features [mt*128 + 64 r, +64) of the gate half (and,
        // 128 rows on, of the up half) of the group's [gate 128 | up 128] blocks
        const int a_row = GU ? t.g * p.a_rows_per_group + t.mt * 2 * kBM + static_cast<int>(rank) * 64
                             : t.g * p.a_rows_per_group + t.mt * 2 * kBM + static_cast<int>(rank) * kBM;
        const uint32_t cta_bytes = narrow ? S::BYTES_N : S::BYTES_W;
        const uint32_t b_off = narrow ? S::B_OFF_N : S::B_OFF_W;
        const uint64_t pol_a = t.nch > 1 ? pol_normal : pol_first;
        bool ok = true;
        for (int st = 0; st < n_st; ++st) {
          const uint32_t s = it % S::STAGES;
          const uint32_t ph = (it / S::STAGES) & 1u;
          if (!mbar_wait(empty0 + 8 * s, ph ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          // (a last stage past K reads zeros for the missing sub-blocks; their
          // bytes still count, and the issuer skips their MMAs)
          if (rank == 0) mbar_arrive_expect_tx(full0 + 8 * s, 2 * cta_bytes);
          const uint32_t fb = full_leader + 8 * s;
          const uint32_t sa = smem_u32(smem + s * S::STAGE_BYTES);
          const int kb0 = st * ks;
          if (GU)
            tma_load_4d_pair(sa, ma, fb, 0, a_row, 0, kb0, pol_a);
          else
            tma_load_3d_pair(sa, ma, fb, 0, a_row, kb0, pol_a);
          tma_load_3d_pair(sa + b_off, mb, fb, 0, b_row, kb0, pol_b);
          ++it;
        }
        if (!ok) break;
      }
      // the leader sees every armed stage land (both CTAs' bytes complete on
      // its barriers); the peer is held by the cluster barrier at the end
      if (rank == 0) {
        const uint32_t used = it < static_cast<uint32_t>(S::STAGES) ? it : S::STAGES;
        for (uint32_t s = 0; s < used; ++s) {
          const uint32_t last = (it - 1u) - ((it - 1u - s) % S::STAGES);
          mbar_wait(full0 + 8 * s, (last / S::STAGES) & 1u, nullptr, p.status);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (rank == 0 && lane == 0) {
      const uint64_t desc0 = sdesc_k_sw<128>(smem_u32(smem));
      uint32_t it = 0, tc = 0;
      for (int w = pair; w < total; w += n_pairs) {
        if (*abort_flag) break;
        const Tile t = decode_tile<BN>(gp, w);
        const int n_mma = (t.n_valid + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(2 * kBM, n_mma);
        const uint32_t buf = tc & 1u;
        const uint32_t tph = (tc >> 1) & 1u;
        if (!mbar_wait(tempty0 + 8 * buf, tph ^ 1u, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + buf * S::ACC_COLS;
        const bool narrow = narrow_tile(t.n_valid);
        const int ks = narrow ? S::KS_N : S::KS_W;
        const int n_st = (p.num_kb + ks - 1) / ks;
        const uint32_t b_off = narrow ? S::B_OFF_N : S::B_OFF_W;
        bool ok = true;
        for (int st = 0; st < n_st; ++st) {
          const uint32_t s = it % S::STAGES;
          const uint32_t ph = (it / S::STAGES) & 1u;
          if (!mbar_wait(full0 + 8 * s, ph, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = desc0 + static_cast<uint64_t>((s * S::STAGE_BYTES) >> 4);
          const uint64_t bd = ad + static_cast<uint64_t>(b_off >> 4);
          const int nsub = min(ks, p.num_kb - st * ks);  // K sub-blocks inside K
          if (narrow)
            issue_stage_pair<S::KS_N, S::SUB_A, S::SUB_BN>(d, ad, bd, idesc, nsub, st == 0);
          else
            issue_stage_pair<S::KS_W, S::SUB_A, S::SUB_BW>(d, ad, bd, idesc, nsub, st == 0);
          tc_commit_pair_mc(empty0 + 8 * s, 3);  // frees the stage in both CTAs
          ++it;
        }
        if (!ok) break;
        tc_commit_pair_mc(tfull0 + 8 * buf, 3);  // accumulators ready in both CTAs
        ++tc;
      }
      if (it > 0) {  // no MMA may still be writing TMEM at deallocation
        tc_commit_pair(drain);
        mbar_wait(drain, 0, nullptr, p.status);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // the TMEM lane quadrant this warp may read
    const int ew = warp - 2;
    uint8_t* stg_base = smem + S::EPI_OFFSET + ew * 2 * S::STG_BYTES;
    const uint32_t tempty_leader = mapa_shared(tempty0, 0);
    uint32_t chunks = 0;  // output chunks this warp has staged (double buffer index)
    if (lane == 0) prefetch_tmap(&tmOut);
    float* wbuf = reinterpret_cast<float*>(smem + S::WB_OFFSET) + ew * BN;
    uint32_t tc = 0;
    for (int w = pair; w < total; w += n_pairs) {
      const Tile t = decode_tile<BN>(gp, w);
      const uint32_t buf = tc & 1u;
      const uint32_t tph = (tc >> 1) & 1u;
      const size_t row0 = static_cast<size_t>(group_row0(gp, t.g)) + static_cast<size_t>(t.nc) * BN;
      // down: the tile's gate weights, loaded while the accumulators are computed
      float wl[BN / 32];
      if (!GU) {
#pragma unroll
        for (int m = 0; m < BN / 32; ++m)
          wl[m] = lane + 32 * m < t.n_valid ? __ldg(p.w_perm + row0 + lane + 32 * m) : 0.f;
      }
      int ok = 1;
      if (lane == 0) ok = mbar_wait(tfull0 + 8 * buf, tph, abort_flag, p.status) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (GU) {
        // the two warps of a gate|up pair meet at named barriers, so they
        // continue or stop together (slot by tile parity: a slot is written
        // again only after both warps have passed another barrier)
        volatile int* okx = reinterpret_cast<volatile int*>(smem + S::OKX_OFFSET) +
                            (q & 1) * 4 + (tc & 1u) * 2;
        if (lane == 0) okx[q < 2 ? 0 : 1] = ok;
        named_bar_sync(1 + (q & 1), 64);
        ok = okx[0] & okx[1];
      }
      if (!ok) break;
      tc_fence_after();
      if (!GU) {
#pragma unroll
        for (int m = 0; m < BN / 32; ++m) wbuf[lane + 32 * m] = wl[m];
        __syncwarp();
      }
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * S::ACC_COLS;
      if (GU) {
        // lanes 0-63 gate, 64-127 up of features [mt*128 + 64 r, +64): warp q
        // (gate, q < 2) and warp q + 2 (up) share features fbase + lane; the
        // gate warp finishes tokens 0-7 of each 16-token chunk, the up warp
        // tokens 8-15
        const bool is_gate = q < 2;
        const int pr = q & 1;
        const uint32_t bar_id = 1 + pr;
        float* xch = reinterpret_cast<float*>(smem + S::EPI_OFFSET + 4 * 2 * S::STG_BYTES +
                                              pr * S::XCH_BYTES);
        const int fbase = t.mt * kBM + static_cast<int>(rank) * 64 + pr * 32;
        __nv_bfloat16* outp = p.out + row0 * p.out_ld + fbase + lane;
        const float L = (t.g == p.E) ? p.limit_shared : p.limit;
        for (int c0 = 0; c0 < t.n_valid; c0 += kEpiRows) {
          uint32_t ra[16];
          tmem_ld_x16(taddr + c0, ra);
          tmem_ld_wait();
          const bool full = c0 + kEpiRows <= t.n_valid;
          const uint32_t buf_off = (chunks & 1u) * S::STG_BYTES;
          // the gate warp issues the chunk's TMA store: before the staging
          // buffer of two chunks ago is rewritten its store must have read it
          if (full && is_gate && chunks >= 2 && lane == 0) bulk_wait_group_read<1>();
          // hand over the other warp's 8 tokens
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
          const int r0 = is_gate ? 0 : 8;  // this warp's rows of the chunk
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
                outp[static_cast<size_t>(c0 + r0 + i) * p.out_ld] = __float2bfloat16_rn(hv[i]);
          }
          named_bar_sync(bar_id, 64);  // chunk staged; exchange buffer free again
          if (full) {
            if (is_gate && lane == 0) {
              const uint32_t src = smem_u32(smem + S::EPI_OFFSET + (pr * 2) * 2 * S::STG_BYTES +
                                            buf_off);
              tma_store_2d(&tmOut, src, fbase, static_cast<int>(row0) + c0);
              bulk_commit_group();
            }
            ++chunks;
          }
        }
      } else {
        const int feat = t.mt * 2 * kBM + static_cast<int>(rank) * kBM + q * 32 + lane;
        __nv_bfloat16* outp = p.out + row0 * p.out_ld + feat;
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
              tma_store_2d(&tmOut, smem_u32(stg), feat - lane, static_cast<int>(row0) + c0);
              bulk_commit_group();
            }
            ++chunks;
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (c0 + i < t.n_valid)
                outp[static_cast<size_t>(c0 + i) * p.out_ld] =
                    __float2bfloat16_rn(__uint_as_float(ra[i]) * wv[i]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader + 8 * buf);
      ++tc;
    }
    if (lane == 0) bulk_wait_group_all();  // h / y fully written
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

using GuPair = PairShape<kModeGateUp>;
using DnPair = PairShape<kModeDown>;

int g_pair_grid = 0;  // CTAs per launch: twice the co-resident clusters

}  // namespace

cudaError_t gemm_pair_configure_device(int num_sms) {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(grouped_gemm_pair_kernel<kModeGateUp>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(GuPair::SMEM))) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(grouped_gemm_pair_kernel<kModeDown>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(DnPair::SMEM))) != cudaSuccess)
    return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms & ~1), 1, 1);
  cfg.blockDim = dim3(GuPair::THREADS, 1, 1);
  cfg.dynamicSmemBytes = GuPair::SMEM;
  cudaLaunchAttribute attr{};
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if ((e = cudaOccupancyMaxActiveClusters(&clusters, grouped_gemm_pair_kernel<kModeGateUp>,
                                          &cfg)) != cudaSuccess)
    return e;
  g_pair_grid = 2 * (clusters < num_sms / 2 ? clusters : num_sms / 2);
  return g_pair_grid > 0 ? cudaSuccess : cudaErrorInvalidConfiguration;
}

int gemm_pair_grid() { return g_pair_grid; }

cudaError_t launch_gemm_gate_up_pair(const GemmMaps& m, const GemmParams& p, cudaStream_t st) {
  if (g_pair_grid <= 0) return cudaErrorInvalidConfiguration;
  return launch_pdl(grouped_gemm_pair_kernel<kModeGateUp>, dim3(g_pair_grid),
                    dim3(GuPair::THREADS), GuPair::SMEM, st, m.a, m.a2, m.b, m.bsh, m.bw, m.bshw,
                    m.out, p);
}

cudaError_t launch_gemm_down_pair(const GemmMaps& m, const GemmParams& p, cudaStream_t st) {
  if (g_pair_grid <= 0) return cudaErrorInvalidConfiguration;
  return launch_pdl(grouped_gemm_pair_kernel<kModeDown>, dim3(g_pair_grid),
                    dim3(DnPair::THREADS), DnPair::SMEM, st, m.a, m.a2, m.b, m.b, m.bw, m.bw, m.out,
                    p);
}

}  // namespace moe
