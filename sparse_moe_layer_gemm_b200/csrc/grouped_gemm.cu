// K5 / K6: grouped GEMMs of the routed experts plus the shared expert (group
// E, an always-on 289th group), on the 5th-generation tensor cores.
//
//   K5 (gate|up):  for group g and its rows X_g:  a = X_g . Wg_g, u = X_g . Wu_g,
//                  optional clamp (gate = min(a, L), up = clip(u, -L, L)),
//                  h = silu(gate) * up, stored bf16.
//   K6 (down):     y = (h_g . Wd_g) * w_row, the row's gate weight (1 for the
//                  shared rows), stored bf16.
//   split-K partials (dense MLP at small T): part z of a single group's
//                  product over K slice z, raw fp32 accumulators per packed
//                  weight row; a reduction kernel finishes the layer.
//   fp32 expert path (fp32 weights): the same K5 / K6 on the tf32 tensor cores
//                  over the three-term split of tf32.cuh, h and y kept fp32.
//   K1 (router, large T):  logits = x . W_r on the bf16 tensor cores: W_r =
//                  W1 + W2 + W3 split into three bf16 terms concatenated along
//                  K; the tiles of part z accumulate x . Wz (each bf16 x bf16
//                  product is exact in fp32; x is bf16) and store it, fp32,
//                  as partial z; the top-k adds the three parts.
//
// The expert FFN is the SwiGLU of sglang-jax issue #1367 "Support Step 3.5
// Flash", section "Model configuration" (MoE bullet; clamped SwiGLU via
// swiglu_limits, 0.0 meaning no clamp) and section "Reuse map" (SiLU-and-mul
// with an elementwise clamp branch); sizes from llm-atlas "Step-3.5-Flash",
// "Raw config fields" (moe_intermediate_size 1280, share_expert_dim 1280).
//
// Design (swap-AB): the MMA's M side (128) is always a block of weight rows,
// the N side the group's tokens (rounded up to 16, at most 128 per tile), so
// ragged groups of 1..21 tokens (decode) waste no more than 15 columns.
// A tile is (group, weight tile mt, token block nc); the order of a group's
// tiles (chunks of token blocks, weight-tile major inside a chunk) is
// described at decode_tile.
//
// One persistent CTA per SM, 4 + NI warps:
//   warp 0        TMA producer: per stage one box of the tile's weight rows
//                 (BLOCKS 128-feature blocks; gate|up blocks are 128 gate rows
//                 then 128 up rows) x 64 K and one box of token rows (32 rows
//                 for tiles of <= 32 tokens, else 128), 128-byte swizzle.
//   warps 1..NI   tcgen05.mma issuers (kind::f16, bf16 x bf16 -> fp32 TMEM;
//                 the fp32 path kind::tf32 on the same 128-byte rows):
//                 each owns every NI-th 128-row accumulator of the tile (gate
//                 and up, or two weight blocks) and keeps its own stage waits
//                 and commits, so the issue latencies of the accumulator
//                 chains overlap; warp 1 also allocates TMEM.  Two
//                 accumulator buffers let the epilogue of tile i overlap the
//                 mainloop of tile i+1.
//   last 4 warps  epilogue: tcgen05.ld (32 lanes x 16 columns), SwiGLU or
//                 gate weight in registers, bf16 (router: fp32) stores.
// No TMA multicast anywhere.
#include "gemm_common.cuh"
#include "moe_internal.h"
#include "moe_ptx.cuh"
#include "tf32.cuh"

namespace moe {

namespace {

using namespace gemm;

// Tile shape: BLOCKS weight blocks of 128 features per tile (gate|up: each
// block is 128 gate rows + 128 up rows), BN tokens per tile, one 128-byte
// swizzled row of reduction elements per pipeline stage: BK = 64 bf16, or 32
// fp32 for the tf32 path (TF).  Either way a stage row takes four MMAs of 32
// bytes of K (16 bf16 or 8 tf32 elements).
template <int MODE, int BLOCKS, int BN_, bool TF_ = false>
struct Shape {
  static constexpr bool TF = TF_;
  static constexpr bool GU = MODE == kModeGateUp;
  // router with BLOCKS = 2: one weight block, the tile's tokens split into two
  // halves, one accumulator (and issuer) each
  static constexpr bool TOKSPLIT = MODE == kModeRouter && BLOCKS == 2;
  // fp32 outputs straight from the accumulators (no tables, no TMA stores)
  static constexpr bool F32OUT = MODE == kModeRouter || MODE == kModePartial;
  static constexpr int BN = BN_;
  static constexpr int BK = TF ? kBK32 : kBK;
  static constexpr int ROW = 128;                           // bytes per operand row in SMEM
  static constexpr int ACCS = BLOCKS * (GU ? 2 : 1);       // 128-row accumulators per tile
  static constexpr int NI = ACCS >= 2 ? 2 : 1;             // MMA-issuing warps
  static constexpr int THREADS = 32 * (1 + NI + 4);
  static constexpr int A_ROWS = TOKSPLIT ? kBM : kBM * ACCS;
  static constexpr int ACC_N = TOKSPLIT ? BN / 2 : BN;      // tokens (columns) per accumulator
  static constexpr int A_BOX = GU ? 2 * kBM : kBM;         // rows per A box (the tensor maps')
  static constexpr int A_LOADS = A_ROWS / A_BOX;
  static constexpr int A_BYTES = A_ROWS * ROW;
  static constexpr int B_BYTES = BN * ROW;
  static constexpr int B_BOX_BYTES = kBBoxRows * ROW;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (200 * 1024 / STAGE_BYTES) < 6 ? (200 * 1024 / STAGE_BYTES) : 6;
  static constexpr int ACC_COLS = ACCS * ACC_N;             // TMEM columns per accumulator buffer
  static constexpr int NBUF = ACC_COLS <= 256 ? 2 : 1;     // double-buffered when it fits
  static constexpr int TMEM_COLS = NBUF * ACC_COLS > 256 ? 512 : 256;
  static constexpr int BAR_BYTES = 256;
  // gate|up and down epilogues: per epilogue warp two 16-row x 32-feature
  // bf16 staging buffers for TMA stores of h or y
  // (down: plus per warp the tile's BN gate weights, fp32)
  static constexpr int EPI_STAGE_BYTES =
      !F32OUT ? 4 * 2 * kEpiRows * 32 * 2 + (MODE == kModeDown ? 4 * BN * 4 : 0) : 0;
  // group tables (tile_start, counts, row_start) copied to shared memory
  static constexpr int TAB_OFFSET = STAGES * STAGE_BYTES + BAR_BYTES + EPI_STAGE_BYTES;
  static constexpr int TAB_BYTES = !F32OUT ? kTabBytes : 0;
  static constexpr size_t SMEM = 1024 + static_cast<size_t>(TAB_OFFSET) + TAB_BYTES;
  static_assert((2 * STAGES + 5) * 8 + 8 <= BAR_BYTES, "barrier area");
  static_assert(NBUF * ACC_COLS <= 512, "TMEM capacity");
  static_assert(BN % kBN == 0, "token tile: whole wide (kBN-row) token-row boxes");
  static_assert(A_ROWS % A_BOX == 0 && ACCS % NI == 0, "A boxes, issuer split");
  static_assert(STAGES >= 2, "pipeline depth");
  static_assert(STAGE_BYTES % 1024 == 0 && A_BYTES % 1024 == 0, "swizzle atoms stay aligned");
  // descriptor start-address field: 14 bits of (address >> 4), no carries
  static_assert(1024 + STAGES * STAGE_BYTES + BAR_BYTES <= 256 * 1024, "descriptor range");
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
  static_assert(!TF || MODE == kModeGateUp || MODE == kModeDown, "tf32: expert GEMMs only");
};

// tcgen05.mma issue without a memory clobber: the MMA reads shared memory
// the TMA wrote (ordered by the full-barrier wait and the tcgen05 fence) and
// writes TMEM; its completion is ordered by the (volatile, clobbering)
// commit that follows it.
template <bool TF>
__device__ __forceinline__ void mma_issue(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  if (TF)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// tmB / tmBsh: token-row operands with kBBoxRows-row boxes; tmBw / tmBshw
// the same tensors with BN-row boxes, used when a tile has more than
// kBBoxRows tokens (one TMA instruction per stage instead of several).
template <int MODE, int BLOCKS, int BN, bool TF>
__global__ void __launch_bounds__(Shape<MODE, BLOCKS, BN, TF>::THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmBsh,
                        const __grid_constant__ CUtensorMap tmBw,
                        const __grid_constant__ CUtensorMap tmBshw,
                        const __grid_constant__ CUtensorMap tmOut, const GemmParams p) {
  using S = Shape<MODE, BLOCKS, BN, TF>;
  constexpr bool GU = S::GU;
  constexpr int BK = S::BK;
  extern __shared__ uint8_t smem_raw[];
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

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, S::NI);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, S::NI);
      mbar_init(tempty0 + 8 * b, 4);
    }
    mbar_init(drain, S::NI);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmBw);
    if (GU) {
      prefetch_tmap(&tmBsh);
      prefetch_tmap(&tmBshw);
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), S::TMEM_COLS);
    tmem_relinquish();
  }
  // everything above touched only this CTA's resources; from here on the
  // previous kernel's outputs are read
  pdl_wait();
  // group tables in shared memory (visible after the __syncthreads below)
  const GemmParams gp =
      !S::F32OUT ? stage_group_tables(p, reinterpret_cast<int*>(smem + S::TAB_OFFSET)) : p;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = total_tiles<BN>(gp);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // weights: evict-first when only one token block reads them, else
      // normal so the other token blocks of the group find them in L2;
      // token rows: evict-last, every weight tile of the chunk reads them
      const uint64_t pol_first = l2_policy_evict_first();
      const uint64_t pol_normal = l2_policy_evict_normal();
      const uint64_t pol_b = l2_policy_evict_last();
      uint32_t it = 0;
      for (int w = blockIdx.x; w < total; w += gridDim.x) {
        if (*abort_flag) break;
        const Tile t = decode_tile<BN>(gp, w);
        const int n_mma = (t.n_valid + 15) & ~15;
        // token rows: kBN-row boxes (as many as the MMA's N needs), else one
        // kBBoxRows-row box
        const bool wide = n_mma > kBBoxRows;
        const int nbox = wide ? (n_mma + kBN - 1) / kBN : 1;
        const bool sh = GU && t.g == p.E;
        const CUtensorMap* mb = wide ? (sh ? &tmBshw : &tmBw) : (sh ? &tmBsh : &tmB);
        const int b_row = (sh ? p.shared_b_row0 : group_row0(gp, t.g)) + t.nc * BN;
        const int a_row = t.g * p.a_rows_per_group + t.mt * S::A_ROWS;
        const uint32_t bytes = S::A_BYTES + (wide ? nbox * kBN * S::ROW : S::B_BOX_BYTES);
        const uint64_t pol_a = t.nch > 1 ? pol_normal : pol_first;
        const int a_k0 = t.kz * p.num_kb * BK;  // K part of a split-K tile
        // router: every part multiplies the same token rows (the parts are
        // terms of W_r); split-K partials: the token rows' own K slice
        const int b_k0 = MODE == kModePartial ? a_k0 : 0;
        bool ok = true;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          const uint32_t s = it % S::STAGES;
          const uint32_t ph = (it / S::STAGES) & 1u;
          if (!mbar_wait(empty0 + 8 * s, ph ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          // K columns of this stage; the tf32 path's terms hi.hi, lo.hi,
          // hi.lo read the lo half (kb_term k-blocks in) of A, resp. B
          int ak = a_k0 + kb * BK, bk = b_k0 + kb * BK;
          if (TF) {
            const int term = kb / p.kb_term;
            const int kk = (kb - term * p.kb_term) * BK;
            ak = (term == 1 ? p.kb_term * BK : 0) + kk;
            bk = (term == 2 ? p.kb_term * BK : 0) + kk;
          }
          const uint32_t fb = full0 + 8 * s;
          mbar_arrive_expect_tx(fb, bytes);
          const uint32_t sa = smem_u32(smem + s * S::STAGE_BYTES);
#pragma unroll
          for (int i = 0; i < S::A_LOADS; ++i)
            tma_load_2d(sa + i * S::A_BOX * S::ROW, &tmA, fb, ak, a_row + i * S::A_BOX, pol_a);
          for (int i = 0; i < nbox; ++i)
            tma_load_2d(sa + S::A_BYTES + i * kBN * S::ROW, mb, fb, bk, b_row + i * kBN, pol_b);
          ++it;
        }
        if (!ok) break;
      }
      // every armed stage must have landed before the CTA may exit
      const uint32_t used = it < static_cast<uint32_t>(S::STAGES) ? it : S::STAGES;
      for (uint32_t s = 0; s < used; ++s) {
        const uint32_t last = (it - 1u) - ((it - 1u - s) % S::STAGES);
        mbar_wait(full0 + 8 * s, (last / S::STAGES) & 1u, nullptr, p.status);
      }
    }
  } else if (warp <= S::NI) {
    // ------------------------------------------------------------ MMA issuers
    if (lane == 0) {
      const int me = warp - 1;  // this warp issues accumulators me, me + NI, ...
      const uint64_t desc0 = sdesc_k_sw<S::ROW>(smem_u32(smem));
      uint32_t it = 0, tc = 0;
      for (int w = blockIdx.x; w < total; w += gridDim.x) {
        if (*abort_flag) break;
        const Tile t = decode_tile<BN>(gp, w);
        // token-split router tiles: this issuer's half of the tokens (none
        // for a ragged tile's empty second half: it only commits)
        const int n_me = S::TOKSPLIT ? min(S::ACC_N, max(0, t.n_valid - me * S::ACC_N)) : t.n_valid;
        const int n_mma = (n_me + 15) & ~15;
        const uint32_t idesc = TF ? idesc_tf32_f32(kBM, n_mma > 0 ? n_mma : 16)
                                  : idesc_bf16_f32(kBM, n_mma > 0 ? n_mma : 16);
        const uint32_t buf = S::NBUF == 2 ? (tc & 1u) : 0u;
        const uint32_t tph = (S::NBUF == 2 ? (tc >> 1) : tc) & 1u;
        if (!mbar_wait(tempty0 + 8 * buf, tph ^ 1u, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + buf * S::ACC_COLS;
        bool ok = true;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          const uint32_t s = it % S::STAGES;
          const uint32_t ph = (it / S::STAGES) & 1u;
          if (!mbar_wait(full0 + 8 * s, ph, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // stage descriptors: the start field advances by (byte offset >> 4)
          const uint64_t ad = desc0 + static_cast<uint64_t>((s * S::STAGE_BYTES) >> 4);
          const uint64_t bd = ad + static_cast<uint64_t>(S::A_BYTES >> 4);
          const uint32_t acc0 = kb != 0 ? 1u : 0u;
          if (n_mma > 0) {
#pragma unroll
            for (int kk = 0; kk < S::ROW / 32; ++kk)
#pragma unroll
              for (int j = 0; j < S::ACCS / S::NI; ++j) {
                const int a = j * S::NI + me;
                // accumulator a: its own weight rows, or (token split) its
                // own half of the token rows
                const int a_off = S::TOKSPLIT ? 0 : a * kBM * S::ROW;
                const int b_off = S::TOKSPLIT ? a * S::ACC_N * S::ROW : 0;
                mma_issue<TF>(d + a * S::ACC_N, ad + static_cast<uint64_t>((a_off + kk * 32) >> 4),
                          bd + static_cast<uint64_t>((b_off + kk * 32) >> 4), idesc,
                          kk == 0 ? acc0 : 1u);
              }
          }
          tc_commit(empty0 + 8 * s);  // frees the stage once these MMAs have read it
          ++it;
        }
        if (!ok) break;
        tc_commit(tfull0 + 8 * buf);  // this warp's accumulators are ready
        ++tc;
      }
      if (it > 0) {  // no MMA may still be writing TMEM at deallocation
        tc_commit(drain);
        mbar_wait(drain, 0, nullptr, p.status);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // the TMEM lane quadrant this warp may read
    // this warp's two output staging buffers (16 rows x 32 features bf16)
    uint8_t* epi_stage = smem + S::STAGES * S::STAGE_BYTES + S::BAR_BYTES +
                         (warp - (1 + S::NI)) * 2 * kEpiRows * 32 * 2;
    // down: the tile's gate weights, loaded once per tile while the
    // accumulators are still being computed
    float* wbuf = reinterpret_cast<float*>(smem + S::STAGES * S::STAGE_BYTES + S::BAR_BYTES +
                                           4 * 2 * kEpiRows * 32 * 2) +
                  (warp - (1 + S::NI)) * BN;
    uint32_t chunks = 0;  // TMA-store chunks this warp has issued
    if (!S::F32OUT && !TF && lane == 0) prefetch_tmap(&tmOut);
    // Writes rows [c0, c0 + 16) of this lane's output feature.  A chunk whose
    // 16 rows all belong to the tile goes through a staging buffer and one
    // TMA store of 16 x 32 values; a ragged one is stored directly, so no row
    // of another group is ever written.
    auto store_chunk = [&](const float (&v)[16], int c0, int n_valid, size_t row0, int feat,
                           __nv_bfloat16* outp) {
      if (c0 + kEpiRows <= n_valid) {
        const uint32_t buf_off = (chunks & 1u) * (kEpiRows * 32 * 2);
        if (chunks >= 2 && lane == 0) bulk_wait_group_read<1>();  // buffer free again
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
      float wl[BN / 32];
      if (MODE == kModeDown) {
#pragma unroll
        for (int m = 0; m < BN / 32; ++m)
          wl[m] = lane + 32 * m < t.n_valid ? __ldg(p.w_perm + row0 + lane + 32 * m) : 0.f;
      }
      int ok = 1;
      if (lane == 0) ok = mbar_wait(tfull0 + 8 * buf, tph, abort_flag, p.status) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      if (MODE == kModeDown) {
#pragma unroll
        for (int m = 0; m < BN / 32; ++m) wbuf[lane + 32 * m] = wl[m];
        __syncwarp();
      }
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * S::ACC_COLS;
#pragma unroll 1
      for (int b = 0; b < BLOCKS; ++b) {
        const int fblock = S::TOKSPLIT ? t.mt : t.mt * BLOCKS + b;  // 128-feature block
        const int feat = fblock * kBM + q * 32 + lane;
        if (fblock * kBM >= p.out_feats) break;  // never past the output
        if (MODE == kModePartial) {
          // raw accumulators of packed weight row prow for the tile's tokens
          const int prow = fblock * kBM + q * 32 + lane;
          float* pp = p.out_f32 + t.kz * p.part_stride + row0 * p.out_ld + prow;
          for (int c0 = 0; c0 < t.n_valid; c0 += 16) {
            uint32_t ra[16];
            tmem_ld_x16(taddr + b * BN + c0, ra);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (c0 + i < t.n_valid) pp[static_cast<size_t>(c0 + i) * p.out_ld] = __uint_as_float(ra[i]);
          }
        } else if (MODE == kModeRouter) {
          // token split: accumulator b holds tokens [b * ACC_N, (b + 1) * ACC_N)
          const int tok0 = S::TOKSPLIT ? b * S::ACC_N : 0;
          const int n_b = S::TOKSPLIT ? min(S::ACC_N, t.n_valid - tok0) : t.n_valid;
          float* lp = p.out_f32 + t.kz * p.part_stride + (row0 + tok0) * p.out_ld + feat;
          const bool keep = feat < p.valid_feats;
          for (int c0 = 0; c0 < n_b; c0 += 16) {
            uint32_t ra[16];
            tmem_ld_x16(taddr + b * S::ACC_N + c0, ra);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (keep && c0 + i < n_b)
                lp[static_cast<size_t>(c0 + i) * p.out_ld] = __uint_as_float(ra[i]);
          }
        } else if (GU && TF) {
          // h fp32 as its tf32 split: hi in columns [0, ld / 2), lo after
          float* hp = p.out_f32 + row0 * p.out_ld + feat;
          const int lo_off = p.out_ld / 2;
          const float L = (t.g == p.E) ? p.limit_shared : p.limit;
          const uint32_t tg = taddr + (2 * b) * BN, tu = taddr + (2 * b + 1) * BN;
          for (int c0 = 0; c0 < t.n_valid; c0 += 16) {
            uint32_t ra[16], rb[16];
            tmem_ld_x16(tg + c0, ra);
            tmem_ld_x16(tu + c0, rb);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float a = __uint_as_float(ra[i]);
              float u = __uint_as_float(rb[i]);
              if (L > 0.f) {
                a = fminf(a, L);
                u = fminf(fmaxf(u, -L), L);
              }
              float hi, lo;
              tf32_split(a / (1.0f + expf(-a)) * u, hi, lo);
              if (c0 + i < t.n_valid) {
                hp[static_cast<size_t>(c0 + i) * p.out_ld] = hi;
                hp[static_cast<size_t>(c0 + i) * p.out_ld + lo_off] = lo;
              }
            }
          }
        } else if (TF) {
          // y fp32
          float* yp = p.out_f32 + row0 * p.out_ld + feat;
          for (int c0 = 0; c0 < t.n_valid; c0 += 16) {
            uint32_t ra[16];
            tmem_ld_x16(taddr + b * BN + c0, ra);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (c0 + i < t.n_valid)
                yp[static_cast<size_t>(c0 + i) * p.out_ld] = __uint_as_float(ra[i]) * wbuf[c0 + i];
          }
        } else if (GU) {
          __nv_bfloat16* outp = p.out + row0 * p.out_ld + feat;
          const float L = (t.g == p.E) ? p.limit_shared : p.limit;
          const uint32_t tg = taddr + (2 * b) * BN, tu = taddr + (2 * b + 1) * BN;
          for (int c0 = 0; c0 < t.n_valid; c0 += 16) {
            uint32_t ra[16], rb[16];
            tmem_ld_x16(tg + c0, ra);
            tmem_ld_x16(tu + c0, rb);
            tmem_ld_wait();
            float hv[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float a = __uint_as_float(ra[i]);
              float u = __uint_as_float(rb[i]);
              if (L > 0.f) {
                a = fminf(a, L);
                u = fminf(fmaxf(u, -L), L);
              }
              hv[i] = a / (1.0f + __expf(-a)) * u;
            }
            store_chunk(hv, c0, t.n_valid, row0, feat, outp);
          }
        } else {
          __nv_bfloat16* outp = p.out + row0 * p.out_ld + feat;
          for (int c0 = 0; c0 < t.n_valid; c0 += 16) {
            uint32_t ra[16];
            tmem_ld_x16(taddr + b * BN + c0, ra);
            tmem_ld_wait();
            float yv[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) yv[i] = __uint_as_float(ra[i]) * wbuf[c0 + i];
            store_chunk(yv, c0, t.n_valid, row0, feat, outp);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * buf);
      ++tc;
    }
    if (!S::F32OUT && !TF && lane == 0) bulk_wait_group_all();  // h / y fully written
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, S::TMEM_COLS);
  }
}

// The launch configurations.  gate|up: one 128-feature block per tile (the
// gate and up accumulators, one issuer warp each).  down: two 128-feature
// blocks per tile when H allows (one issuer warp each; double-buffered
// TMEM), else one.  router: one block.
using GuCfg = Shape<kModeGateUp, 1, 128>;
using DnCfg2 = Shape<kModeDown, 2, 128>;
using DnCfg1 = Shape<kModeDown, 1, 128>;
using RtCfg = Shape<kModeRouter, 2, 256>;  // 256-token tiles, one accumulator per half
using PtCfg = Shape<kModePartial, 2, 128>;  // two 128-row blocks, 128-token tiles
// the fp32 path: the gate|up and down configurations on tf32
using GuCfgTf = Shape<kModeGateUp, 1, 128, true>;
using DnCfg2Tf = Shape<kModeDown, 2, 128, true>;
using DnCfg1Tf = Shape<kModeDown, 1, 128, true>;

template <typename S, int MODE, int BLOCKS>
cudaError_t set_smem() {
  return cudaFuncSetAttribute(grouped_gemm_kernel<MODE, BLOCKS, S::BN, S::TF>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(S::SMEM));
}

}  // namespace

cudaError_t gemm_configure_device() {
  cudaError_t e;
  if ((e = set_smem<GuCfg, kModeGateUp, 1>()) != cudaSuccess) return e;
  if ((e = set_smem<DnCfg2, kModeDown, 2>()) != cudaSuccess) return e;
  if ((e = set_smem<DnCfg1, kModeDown, 1>()) != cudaSuccess) return e;
  if ((e = set_smem<PtCfg, kModePartial, 2>()) != cudaSuccess) return e;
  if ((e = set_smem<GuCfgTf, kModeGateUp, 1>()) != cudaSuccess) return e;
  if ((e = set_smem<DnCfg2Tf, kModeDown, 2>()) != cudaSuccess) return e;
  if ((e = set_smem<DnCfg1Tf, kModeDown, 1>()) != cudaSuccess) return e;
  return set_smem<RtCfg, kModeRouter, 2>();
}

int gemm_down_blocks(int H) { return (H / kBM) % 2 == 0 ? 2 : 1; }

cudaError_t launch_gemm_gate_up(const GemmMaps& m, const GemmParams& p, int grid, cudaStream_t st) {
  return launch_pdl(grouped_gemm_kernel<kModeGateUp, 1, 128, false>, dim3(grid), dim3(GuCfg::THREADS),
                    GuCfg::SMEM, st, m.a, m.b, m.bsh, m.bw, m.bshw, m.out, p);
}

cudaError_t launch_gemm_down(const GemmMaps& m, const GemmParams& p, int grid, int blocks,
                             cudaStream_t st) {
  if (blocks == 2)
    return launch_pdl(grouped_gemm_kernel<kModeDown, 2, 128, false>, dim3(grid), dim3(DnCfg2::THREADS),
                      DnCfg2::SMEM, st, m.a, m.b, m.b, m.bw, m.bw, m.out, p);
  return launch_pdl(grouped_gemm_kernel<kModeDown, 1, 128, false>, dim3(grid), dim3(DnCfg1::THREADS),
                    DnCfg1::SMEM, st, m.a, m.b, m.b, m.bw, m.bw, m.out, p);
}

cudaError_t launch_gemm_gate_up_tf32(const GemmMaps& m, const GemmParams& p, int grid,
                                     cudaStream_t st) {
  return launch_pdl(grouped_gemm_kernel<kModeGateUp, 1, 128, true>, dim3(grid),
                    dim3(GuCfgTf::THREADS), GuCfgTf::SMEM, st, m.a, m.b, m.b, m.bw, m.bw, m.b, p);
}

cudaError_t launch_gemm_down_tf32(const GemmMaps& m, const GemmParams& p, int grid, int blocks,
                                  cudaStream_t st) {
  if (blocks == 2)
    return launch_pdl(grouped_gemm_kernel<kModeDown, 2, 128, true>, dim3(grid),
                      dim3(DnCfg2Tf::THREADS), DnCfg2Tf::SMEM, st, m.a, m.b, m.b, m.bw, m.bw,
                      m.b, p);
  return launch_pdl(grouped_gemm_kernel<kModeDown, 1, 128, true>, dim3(grid),
                    dim3(DnCfg1Tf::THREADS), DnCfg1Tf::SMEM, st, m.a, m.b, m.b, m.bw, m.bw, m.b, p);
}

cudaError_t launch_gemm_router(const GemmMaps& m, const GemmParams& p, int grid, cudaStream_t st) {
  return launch_pdl(grouped_gemm_kernel<kModeRouter, 2, 256, false>, dim3(grid), dim3(RtCfg::THREADS),
                    RtCfg::SMEM, st, m.a, m.b, m.b, m.bw, m.bw, m.out, p);
}

}  // namespace moe

namespace moe {

cudaError_t launch_gemm_partial(const GemmMaps& m, const GemmParams& p, int grid, cudaStream_t st) {
  return launch_pdl(grouped_gemm_kernel<kModePartial, 2, 128, false>, dim3(grid), dim3(PtCfg::THREADS),
                    PtCfg::SMEM, st, m.a, m.b, m.b, m.bw, m.bw, m.out, p);
}

}  // namespace moe
