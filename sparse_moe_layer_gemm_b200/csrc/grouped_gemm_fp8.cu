// K5 / K6 with FP8 E4M3 expert weights: the grouped gate|up + SwiGLU and
// down x gate-weight GEMMs of the routed experts plus the shared one, with the
// weights stored as one E4M3FN code per element and one fp32 scale per output
// feature (w[k][n] = value(code[k][n]) * scale[n]).  What the layer computes
// is the same SwiGLU expert FFN as the bf16 kernels (sglang-jax issue #1367
// "Support Step 3.5 Flash", section "Model configuration", MoE bullet; the
// pages list FP8 official weights in the same bullet list, without a format).
//
// Every finite E4M3 code is exactly a bf16 value, so the codes are expanded to
// bf16 (into tensor memory, below) and multiplied on the same bf16 x bf16 ->
// fp32 tensor-core path; the epilogue multiplies each accumulator row (one
// output feature) by its scale.  HBM moves one byte per weight instead of two.
//
// Swap-AB tiles as in the bf16 kernel (128 weight rows per MMA on M, up to
// kFp8BN tokens on N), one persistent CTA per SM.  The expanded weights never
// touch shared memory: the MMA reads its A operand from tensor memory.
//   shared memory   two rings: RC code slots, each a stage's codes (one
//                   contiguous run of the tile-major layout, one plain bulk
//                   copy), freed by the converters once the codes are in
//                   registers; RB token-row slots, each the tile's rows for
//                   both k-steps (B, bf16, 128-byte swizzle, one 3-D TMA
//                   box), freed by the MMA commits (the MMA reads B there);
//   tensor memory   the partial accumulators (chain x stage parity, BN columns
//                   each; two buffers when they fit in 256 columns), then SA
//                   stages of expanded weights, 64 columns (128 bf16 of K) per
//                   128-row accumulator operand, lane = weight row; smaller
//                   token tiles leave room for more stages.
// Warps:
//   0         code producer (one bulk copy per stage);
//   1         token-row producer (one TMA load per stage);
//   next 2*NI tcgen05.mma issuers: per accumulator chain (gate and up, or
//             two weight blocks) two warps taking alternate stages into two
//             partial accumulators that the epilogue adds, so that each
//             issuer (about a hundred cycles per MMA at these shapes) has
//             two stages of time for one stage's MMAs; the first allocates
//             TMEM;
//   next 8    converters, two groups of four taking alternate stages: thread
//             = one weight row of every chain, 64-byte-swizzled code reads
//             without bank conflicts, E4M3 -> bf16 in registers, tcgen05.st
//             into the stage (each warp writes the TMEM lane quadrant of its
//             warp index % 4);
//   last 4    epilogue: tcgen05.ld, scale, SwiGLU (gate|up) or gate weight
//             (down), bf16 TMA stores.
// A pipeline stage is two k-steps (K = 128): per stage an issuer waits on one
// barrier (its operand stage), issues eight MMAs and two commits, and each
// converter group handles every other stage.  No TMA multicast anywhere.
#include "fp8.cuh"
#include "gemm_common.cuh"
#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {

namespace {

using namespace gemm;

template <int MODE, int BLOCKS>
struct F8Shape {
  static constexpr bool GU = MODE == kModeGateUp;
  static constexpr int BN = kFp8BN;                          // tokens per tile
  static constexpr int BK = kBK;                             // K per k-step (one code block)
  static constexpr int KS = 2;                               // k-steps per pipeline stage
  static constexpr int ROW = BK * 2;                         // bf16 bytes per B row
  static constexpr int ACCS = BLOCKS * (GU ? 2 : 1);         // 128-row accumulators
  static constexpr int NI = ACCS;                            // accumulator chains
  static constexpr int NISS = 2 * NI;                        // issuers: chain x stage parity
  static constexpr int GROUPS = 2;                           // converter groups (4 warps each)
  static constexpr int CONV = 4 * GROUPS;
  static constexpr int W_ISS = 2;
  static constexpr int W_CONV = W_ISS + NISS;
  static constexpr int W_EPI = W_CONV + CONV;
  static constexpr int THREADS = 32 * (W_EPI + 4);
  static constexpr int A_ROWS = kBM * ACCS;
  static constexpr int CODE_BYTES = A_ROWS * BK;             // codes of one k-step
  static constexpr int B_BYTES = BN * ROW;                   // token rows of one k-step
  static constexpr int CSLOT = KS * CODE_BYTES;             // codes of both k-steps
  static constexpr int BSLOT = KS * B_BYTES;                 // token rows, k-block-major
  static constexpr int RB = 4;
  static constexpr int RC_FIT = (200 * 1024 - RB * BSLOT) / CSLOT;
  static constexpr int RC = RC_FIT < 8 ? RC_FIT : 8;
  static constexpr int OFF_B = RC * CSLOT;
  static constexpr int ACC_COLS = ACCS * 2 * BN;             // TMEM columns per buffer
  static constexpr int NBUF = 2 * ACC_COLS <= 256 ? 2 : 1;   // accumulator buffers
  static constexpr int A_COL0 = NBUF * ACC_COLS;             // first operand-stage column
  static constexpr int CHAIN_COLS = KS * BK / 2;             // bf16 pairs of a stage's K
  static constexpr int A_STAGE_COLS = ACCS * CHAIN_COLS;
  static constexpr int SA = (512 - A_COL0) / A_STAGE_COLS;   // operand stages in TMEM
  static constexpr int OFF_BAR = OFF_B + RB * BSLOT;
  static constexpr int NBARS = 2 * RC + 2 * RB + 2 * SA * NI + 5;
  static constexpr int BAR_BYTES = 512;
  static constexpr int OFF_EPI = OFF_BAR + BAR_BYTES;
  static constexpr int EPI_STAGE_BYTES =
      4 * 2 * kEpiRows * 32 * 2 + (MODE == kModeDown ? 4 * BN * 4 : 0);
  static constexpr int TAB_OFFSET = OFF_EPI + EPI_STAGE_BYTES;
  static constexpr size_t SMEM = 1024 + static_cast<size_t>(TAB_OFFSET) + kTabBytes;
  static_assert(MODE == kModeGateUp || MODE == kModeDown, "expert GEMMs");
  static_assert(ACCS == 1 || ACCS == 2, "one or two accumulator chains");
  static_assert(SA >= 2 && A_COL0 + SA * A_STAGE_COLS <= 512, "tensor memory");
  // each converter group must wait on every phase of its stages' barriers in
  // order (a parity wait is ambiguous two phases apart): the groups own
  // disjoint sets of stages
  static_assert(SA % GROUPS == 0, "operand stages per converter group");
  static_assert(RC >= 3, "code ring depth");
  static_assert(NBARS * 8 + 8 <= BAR_BYTES, "barrier area");
  static_assert(CSLOT % 1024 == 0 && B_BYTES % 1024 == 0, "slots stay 1024-byte aligned");
  static_assert(OFF_BAR <= 256 * 1024, "descriptor range of the B operands");
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

// tcgen05.mma with A in tensor memory (lane = row, two bf16 of K per column)
// and B in shared memory.
__device__ __forceinline__ void mma_issue_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// Waits (bounded) in lane 0 and broadcasts the outcome to the warp.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          int* status) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort, status) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// 64 codes of one weight row (one k-step), stored as 16-byte chunks at
// positions c ^ sw, -> 32 bf16 pairs in columns [col, col + 32) of this
// thread's TMEM lane.
__device__ __forceinline__ void expand_row(const uint8_t* row_codes, int sw, uint32_t taddr) {
  uint32_t v[32];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 w4 = *reinterpret_cast<const uint4*>(row_codes + ((c ^ sw) << 4));
    e4m3x4_to_bf16x4(w4.x, v[8 * c + 0], v[8 * c + 1]);
    e4m3x4_to_bf16x4(w4.y, v[8 * c + 2], v[8 * c + 3]);
    e4m3x4_to_bf16x4(w4.z, v[8 * c + 4], v[8 * c + 5]);
    e4m3x4_to_bf16x4(w4.w, v[8 * c + 6], v[8 * c + 7]);
  }
  tmem_st_x32(taddr, v);
}

template <int MODE, int BLOCKS>
__global__ void __launch_bounds__(F8Shape<MODE, BLOCKS>::THREADS, 1)
    grouped_gemm_fp8_kernel(const __grid_constant__ CUtensorMap tmB,
                            const __grid_constant__ CUtensorMap tmBsh,
                            const __grid_constant__ CUtensorMap tmOut, const GemmParams p) {
  using S = F8Shape<MODE, BLOCKS>;
  constexpr bool GU = S::GU;
  constexpr int BN = S::BN;
  constexpr int BK = S::BK;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR);
  const uint32_t cfull0 = smem_u32(bars);           // code slots
  const uint32_t cempty0 = cfull0 + 8 * S::RC;
  const uint32_t bfull0 = cempty0 + 8 * S::RC;      // token-row slots
  const uint32_t bempty0 = bfull0 + 8 * S::RB;
  const uint32_t afull0 = bempty0 + 8 * S::RB;      // [operand stage][chain]
  const uint32_t aempty0 = afull0 + 8 * S::SA * S::NI;
  const uint32_t tfull0 = aempty0 + 8 * S::SA * S::NI;
  const uint32_t tempty0 = tfull0 + 16;
  const uint32_t drain = tempty0 + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + S::NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::RC; ++s) {
      mbar_init(cfull0 + 8 * s, 1);
      mbar_init(cempty0 + 8 * s, 4);       // the stage's converter group
    }
    for (int s = 0; s < S::RB; ++s) {
      mbar_init(bfull0 + 8 * s, 1);
      mbar_init(bempty0 + 8 * s, S::NI);   // both chains' MMAs read the slot
    }
    for (int s = 0; s < S::SA * S::NI; ++s) {
      mbar_init(afull0 + 8 * s, 4);  // the stage's converter group, one warp per quadrant
      mbar_init(aempty0 + 8 * s, 1); // that chain's MMA commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, S::NISS);
      mbar_init(tempty0 + 8 * b, 4);
    }
    mbar_init(drain, S::NISS);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1 && lane == 0) {
    prefetch_tmap(&tmB);
    if (GU) prefetch_tmap(&tmBsh);
  }
  if (warp == S::W_ISS) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  // only this CTA's resources were touched so far; now the previous kernel's
  // outputs (routing tables, token rows) are read
  pdl_wait();
  const GemmParams gp = stage_group_tables(p, reinterpret_cast<int*>(smem + S::TAB_OFFSET));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = total_tiles<BN>(gp);
  const int nstage = p.num_kb / S::KS;  // stages per tile (num_kb is even)

  if (warp == 0) {
    // ------------------------------------------------------------ code producer
    if (lane == 0) {
      const uint64_t pol_first = l2_policy_evict_first();
      const uint64_t pol_normal = l2_policy_evict_normal();
      uint32_t it = 0;
      for (int w = blockIdx.x; w < total; w += gridDim.x) {
        if (*abort_flag) break;
        const Tile t = decode_tile<BN>(gp, w);
        // the tile's run for stage st at byte (tile * nstage + st) * CSLOT
        // (tile-major layout); weights read by one token block only are
        // evict-first
        const size_t tile_run = static_cast<size_t>(t.g) * (p.a_rows_per_group / S::A_ROWS) + t.mt;
        const uint64_t pol = t.nch > 1 ? pol_normal : pol_first;
        bool ok = true;
        for (int st = 0; st < nstage; ++st) {
          const uint32_t s = it % S::RC;
          if (!mbar_wait(cempty0 + 8 * s, ((it / S::RC) & 1u) ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          const uint32_t fb = cfull0 + 8 * s;
          mbar_arrive_expect_tx(fb, S::CSLOT);
          bulk_load_1d_hint(smem_u32(smem + s * S::CSLOT),
                            p.a_codes + (tile_run * nstage + st) * S::CSLOT, S::CSLOT, fb, pol);
          ++it;
        }
        if (!ok) break;
      }
      // every armed slot must have landed before the CTA may exit
      const uint32_t used = it < static_cast<uint32_t>(S::RC) ? it : S::RC;
      for (uint32_t s = 0; s < used; ++s) {
        const uint32_t last = (it - 1u) - ((it - 1u - s) % S::RC);
        mbar_wait(cfull0 + 8 * s, (last / S::RC) & 1u, nullptr, p.status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ token-row producer
    if (lane == 0) {
      const uint64_t pol_b = l2_policy_evict_last();  // every weight tile of the chunk reads them
      uint32_t it = 0;
      for (int w = blockIdx.x; w < total; w += gridDim.x) {
        if (*abort_flag) break;
        const Tile t = decode_tile<BN>(gp, w);
        // BN rows x 2 k-blocks per stage (rows past the group's are read but
        // never used; past the tensor they read as zero)
        const bool sh = GU && t.g == p.E;
        const CUtensorMap* mb = sh ? &tmBsh : &tmB;
        const int b_row = (sh ? p.shared_b_row0 : group_row0(gp, t.g)) + t.nc * BN;
        bool ok = true;
        for (int st = 0; st < nstage; ++st) {
          const uint32_t s = it % S::RB;
          if (!mbar_wait(bempty0 + 8 * s, ((it / S::RB) & 1u) ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          const uint32_t fb = bfull0 + 8 * s;
          mbar_arrive_expect_tx(fb, S::BSLOT);
          tma_load_3d(smem_u32(smem + S::OFF_B + s * S::BSLOT), mb, fb, 0, b_row, st * S::KS, pol_b);
          ++it;
        }
        if (!ok) break;
      }
      const uint32_t used = it < static_cast<uint32_t>(S::RB) ? it : S::RB;
      for (uint32_t s = 0; s < used; ++s) {
        const uint32_t last = (it - 1u) - ((it - 1u - s) % S::RB);
        mbar_wait(bfull0 + 8 * s, (last / S::RB) & 1u, nullptr, p.status);
      }
    }
  } else if (warp < S::W_CONV) {
    // ------------------------------------------------------------ MMA issuers
    if (lane == 0) {
      const int me = (warp - S::W_ISS) % S::NI;                             // chain
      const uint32_t par = static_cast<uint32_t>((warp - S::W_ISS) / S::NI);  // stage parity
      const uint64_t desc0 = sdesc_k_sw<S::ROW>(smem_u32(smem));
      uint32_t it = 0, tc = 0;
      for (int w = blockIdx.x; w < total; w += gridDim.x) {
        if (*abort_flag) break;
        const Tile t = decode_tile<BN>(gp, w);
        const int n_mma = (t.n_valid + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(kBM, n_mma);
        const uint32_t buf = S::NBUF == 2 ? (tc & 1u) : 0u;
        const uint32_t tph = (S::NBUF == 2 ? (tc >> 1) : tc) & 1u;
        if (!mbar_wait(tempty0 + 8 * buf, tph ^ 1u, abort_flag, p.status)) break;
        tc_fence_after();
        // this warp's partial accumulator: stages with it % 2 == par
        const uint32_t d = tmem_base + buf * S::ACC_COLS + (me * 2 + par) * BN;
        bool ok = true, first = true;
        for (int st = 0; st < nstage; ++st) {
          if ((it & 1u) != par) {
            ++it;
            continue;
          }
          const uint32_t rb = it % S::RB, sa = it % S::SA;
          const uint32_t ab = (sa * S::NI + me) * 8;
          // the converters waited for the stage's token rows (and codes)
          // before arriving here
          if (!mbar_wait(afull0 + ab, (it / S::SA) & 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_t = tmem_base + S::A_COL0 + sa * S::A_STAGE_COLS + me * S::CHAIN_COLS;
          const uint64_t bd = desc0 + static_cast<uint64_t>((S::OFF_B + rb * S::BSLOT) >> 4);
#pragma unroll
          for (int kk = 0; kk < S::KS * BK / 16; ++kk)
            mma_issue_ts(d, a_t + kk * 8,
                         bd + static_cast<uint64_t>(((kk / 4) * S::B_BYTES + (kk % 4) * 32) >> 4),
                         idesc, (!first || kk != 0) ? 1u : 0u);
          tc_commit(aempty0 + ab);           // the operand stage is free again
          tc_commit(bempty0 + 8 * rb);       // and (both chains) the token rows
          first = false;
          ++it;
        }
        if (!ok) break;
        tc_commit(tfull0 + 8 * buf);
        ++tc;
      }
      if (it > 0) {  // no MMA may still be writing TMEM at deallocation
        tc_commit(drain);
        mbar_wait(drain, 0, nullptr, p.status);
      }
    }
  } else if (warp < S::W_EPI) {
    // ------------------------------------------------------------ converters
    // Two groups of four warps take alternate stages (group g: stages with
    // it % 2 == g), so one group's barrier waits overlap the other's
    // expansion.  Warp -> TMEM lane quadrant
    // q = warp % 4 (the only lanes it may write); thread -> weight row
    // q * 32 + lane of every chain: per stage it expands KS x 64 codes per
    // chain, read as 16-byte chunks from the blocks (chunk c of row r stored
    // at c ^ ((r / 2) % 4) by the packing: a warp's 32 rows hit 8 different
    // bank groups, 4 wavefronts per 512 bytes).
    const int cw = warp - S::W_CONV;
    const int q = warp & 3;
    const int grp = cw >> 2;
    const int row = q * 32 + lane;  // within each chain's 128-row block
    const int sw = (row >> 1) & 3;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    bool ok = true;
    uint32_t it = 0;  // stage counter shared by all roles
    for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
      for (int st = 0; st < nstage; ++st, ++it) {
        if ((it & 1u) != static_cast<uint32_t>(grp)) continue;
        const uint32_t rc = it % S::RC, rb = it % S::RB, sa = it % S::SA;
        const uint32_t cph = (it / S::RC) & 1u;
        // the codes, and the token rows the MMAs will read (arriving on the
        // operand stages below hands both to the issuers)
        if (!warp_wait(cfull0 + 8 * rc, cph, abort_flag, p.status) ||
            !warp_wait(bfull0 + 8 * rb, (it / S::RB) & 1u, abort_flag, p.status)) {
          ok = false;
          break;
        }
        // each lane's own acquire of the landed codes (that phase cannot
        // advance before this group releases the slot)
        (void)mbar_try_wait(cfull0 + 8 * rc, cph);
        const uint8_t* slot = smem + rc * S::CSLOT;
#pragma unroll
        for (int a = 0; a < S::ACCS; ++a) {
          const uint32_t ab = (sa * S::NI + a) * 8;
          if (!warp_wait(aempty0 + ab, ((it / S::SA) & 1u) ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();  // the stage's previous MMAs are done with it
          const uint32_t col = S::A_COL0 + sa * S::A_STAGE_COLS + a * S::CHAIN_COLS;
#pragma unroll
          for (int h = 0; h < S::KS; ++h)
            expand_row(slot + h * S::CODE_BYTES + a * kBM * BK + row * BK, sw,
                       tmem_base + lane_addr + col + h * (BK / 2));
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(afull0 + ab);
        }
        if (!ok) break;
        // the code slot is refilled by a bulk copy (async proxy): order this
        // warp's generic reads of it before that write, then release it
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(cempty0 + 8 * rc);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // the TMEM lane quadrant this warp may read
    const int ew = warp - S::W_EPI;
    uint8_t* epi_stage = smem + S::OFF_EPI + ew * 2 * kEpiRows * 32 * 2;
    float* wbuf = reinterpret_cast<float*>(smem + S::OFF_EPI + 4 * 2 * kEpiRows * 32 * 2) + ew * BN;
    uint32_t chunks = 0;
    if (lane == 0) prefetch_tmap(&tmOut);
    // rows [c0, c0 + 16) of this lane's feature: full chunks through a
    // staging buffer and one TMA store, a ragged one stored directly
    auto store_chunk = [&](const float (&v)[16], int c0, int n_valid, size_t row0, int feat,
                           __nv_bfloat16* outp) {
      if (c0 + kEpiRows <= n_valid) {
        const uint32_t buf_off = (chunks & 1u) * (kEpiRows * 32 * 2);
        if (chunks >= 2 && lane == 0) bulk_wait_group_read<1>();
        __syncwarp();
        __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(epi_stage + buf_off);
#pragma unroll
        for (int i = 0; i < kEpiRows; ++i) stg[i * 32 + lane] = __float2bfloat16_rn(v[i]);
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
          if (c0 + i < n_valid)
            outp[static_cast<size_t>(c0 + i) * p.out_ld] = __float2bfloat16_rn(v[i]);
      }
    };
    uint32_t tc = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      const Tile t = decode_tile<BN>(gp, w);
      const uint32_t buf = S::NBUF == 2 ? (tc & 1u) : 0u;
      const uint32_t tph = (S::NBUF == 2 ? (tc >> 1) : tc) & 1u;
      const size_t row0 = static_cast<size_t>(group_row0(gp, t.g)) + static_cast<size_t>(t.nc) * BN;
      // this lane's feature scale of each chain: weight rows
      // a_row0 + j * 128 + q * 32 + lane
      const size_t srow = static_cast<size_t>(t.g) * p.a_rows_per_group +
                          static_cast<size_t>(t.mt) * S::A_ROWS + q * 32 + lane;
      const float sc0 = __ldg(p.a_scale + srow);
      const float sc1 = S::ACCS > 1 ? __ldg(p.a_scale + srow + kBM) : 0.f;
      constexpr int WL = (BN + 31) / 32;
      float wl[WL];
      if (MODE == kModeDown) {
#pragma unroll
        for (int m = 0; m < WL; ++m)
          wl[m] = lane + 32 * m < t.n_valid ? __ldg(p.w_perm + row0 + lane + 32 * m) : 0.f;
      }
      if (!warp_wait(tfull0 + 8 * buf, tph, abort_flag, p.status)) break;
      tc_fence_after();
      if (MODE == kModeDown) {
#pragma unroll
        for (int m = 0; m < WL; ++m)
          if (lane + 32 * m < BN) wbuf[lane + 32 * m] = wl[m];
        __syncwarp();
      }
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * S::ACC_COLS;
      // partial accumulators: the one of the tile's first stage parity, plus
      // the other one when the tile has more than one stage
      const uint32_t p0 = (static_cast<uint32_t>(tc) * static_cast<uint32_t>(nstage)) & 1u;
      const bool both = nstage > 1;
#pragma unroll 1
      for (int b = 0; b < BLOCKS; ++b) {
        const int fblock = t.mt * BLOCKS + b;
        const int feat = fblock * kBM + q * 32 + lane;
        if (fblock * kBM >= p.out_feats) break;
        __nv_bfloat16* outp = p.out + row0 * p.out_ld + feat;
        if (GU) {
          const float L = (t.g == p.E) ? p.limit_shared : p.limit;
          // chain 2b (gate) and 2b + 1 (up), partial p at (chain * 2 + p) * BN
          const uint32_t tg = taddr + (4 * b) * BN, tu = taddr + (4 * b + 2) * BN;
          for (int c0 = 0; c0 < t.n_valid; c0 += 16) {
            uint32_t ra[16], rb[16];
            float ga[16], ua[16];
            tmem_ld_x16(tg + p0 * BN + c0, ra);
            tmem_ld_x16(tu + p0 * BN + c0, rb);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              ga[i] = __uint_as_float(ra[i]);
              ua[i] = __uint_as_float(rb[i]);
            }
            if (both) {
              tmem_ld_x16(tg + (p0 ^ 1u) * BN + c0, ra);
              tmem_ld_x16(tu + (p0 ^ 1u) * BN + c0, rb);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                ga[i] += __uint_as_float(ra[i]);
                ua[i] += __uint_as_float(rb[i]);
              }
            }
            float hv[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float a = ga[i] * sc0;
              float u = ua[i] * sc1;
              if (L > 0.f) {
                a = fminf(a, L);
                u = fminf(fmaxf(u, -L), L);
              }
              hv[i] = a / (1.0f + __expf(-a)) * u;
            }
            store_chunk(hv, c0, t.n_valid, row0, feat, outp);
          }
        } else {
          const float scb = b == 0 ? sc0 : sc1;
          const uint32_t tb = taddr + (2 * b) * BN;  // chain b's partials
          for (int c0 = 0; c0 < t.n_valid; c0 += 16) {
            uint32_t ra[16], rc[16];
            tmem_ld_x16(tb + p0 * BN + c0, ra);
            if (both) tmem_ld_x16(tb + (p0 ^ 1u) * BN + c0, rc);
            tmem_ld_wait();
            float yv[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              yv[i] = (__uint_as_float(ra[i]) + (both ? __uint_as_float(rc[i]) : 0.f)) * scb *
                      wbuf[c0 + i];
            store_chunk(yv, c0, t.n_valid, row0, feat, outp);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * buf);
      ++tc;
    }
    if (lane == 0) bulk_wait_group_all();  // h / y fully written
  }

  tc_fence_before();
  __syncthreads();
  if (warp == S::W_ISS) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

using GuF8 = F8Shape<kModeGateUp, 1>;
using DnF8x2 = F8Shape<kModeDown, 2>;
using DnF8x1 = F8Shape<kModeDown, 1>;

template <typename S, int MODE, int BLOCKS>
cudaError_t set_smem_f8() {
  return cudaFuncSetAttribute(grouped_gemm_fp8_kernel<MODE, BLOCKS>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(S::SMEM));
}

}  // namespace

cudaError_t gemm_fp8_configure_device() {
  cudaError_t e;
  if ((e = set_smem_f8<GuF8, kModeGateUp, 1>()) != cudaSuccess) return e;
  if ((e = set_smem_f8<DnF8x2, kModeDown, 2>()) != cudaSuccess) return e;
  return set_smem_f8<DnF8x1, kModeDown, 1>();
}

cudaError_t launch_gemm_gate_up_fp8(const GemmMaps& m, const GemmParams& p, int grid,
                                    cudaStream_t st) {
  return launch_pdl(grouped_gemm_fp8_kernel<kModeGateUp, 1>, dim3(grid), dim3(GuF8::THREADS),
                    GuF8::SMEM, st, m.b, m.bsh, m.out, p);
}

cudaError_t launch_gemm_down_fp8(const GemmMaps& m, const GemmParams& p, int grid, int blocks,
                                 cudaStream_t st) {
  if (blocks == 2)
    return launch_pdl(grouped_gemm_fp8_kernel<kModeDown, 2>, dim3(grid), dim3(DnF8x2::THREADS),
                      DnF8x2::SMEM, st, m.b, m.b, m.out, p);
  return launch_pdl(grouped_gemm_fp8_kernel<kModeDown, 1>, dim3(grid), dim3(DnF8x1::THREADS),
                    DnF8x1::SMEM, st, m.b, m.b, m.out, p);
}

}  // namespace moe
