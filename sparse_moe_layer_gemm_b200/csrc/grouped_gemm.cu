// K5 / K6: grouped GEMMs of the routed experts plus the shared expert (group
// E, an always-on 289th group), on the 5th-generation tensor cores.
//
//   K5 (gate|up):  for group g and its rows X_g:  a = X_g . Wg_g, u = X_g . Wu_g,
//                  optional clamp (gate = min(a, L), up = clip(u, -L, L)),
//                  h = silu(gate) * up, stored bf16.
//   K6 (down):     y = (h_g . Wd_g) * w_row, the row's gate weight (1 for the
//                  shared rows), stored bf16.
//   K1 (router, large T):  logits = x . W_r in fp32 accuracy on the bf16 tensor
//                  cores: W_r = W1 + W2 + W3 split into three bf16 terms that
//                  are concatenated along K, so one accumulation over 3H gives
//                  x.W1 + x.W2 + x.W3 (each bf16 x bf16 product is exact in
//                  fp32; x is bf16 and needs no split); stored fp32.
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
// A tile is (group, weight block mt, token block nc); tiles of one group are
// ordered token-block-major so all weight blocks of the same token block run
// together and an expert's weights stay in L2 across its token blocks.
//
// One persistent CTA per SM, 6 warps:
//   warp 0     TMA producer: A = 128 (down) or 2x128 (gate, up) weight rows
//              x 64 K, B = token rows in 32-row boxes, 128-byte swizzle,
//              multi-stage mbarrier ring.
//   warp 1     TMEM allocator and single-thread tcgen05.mma issuer
//              (kind::f16, bf16 x bf16 -> fp32 in TMEM), two accumulator
//              buffers so the epilogue of tile i overlaps the mainloop of i+1.
//   warps 2-5  epilogue: tcgen05.ld (32 lanes x 16 columns), SwiGLU / gate
//              weight in registers, bf16 stores.
// No TMA multicast anywhere.
#include "moe_internal.h"
#include "moe_ptx.cuh"

namespace moe {

namespace {

template <int MODE>
struct Shape {
  static constexpr bool GU = MODE == kModeGateUp;
  static constexpr int A_ROWS = GU ? 2 * kBM : kBM;
  static constexpr int A_BYTES = A_ROWS * kBK * 2;
  static constexpr int B_BYTES = kBN * kBK * 2;
  static constexpr int B_BOX_BYTES = kBBoxRows * kBK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = GU ? 4 : 6;
  static constexpr int ACC_COLS = GU ? 2 * kBN : kBN;  // TMEM columns per accumulator buffer
  static constexpr int TMEM_COLS = 2 * ACC_COLS;       // two buffers
  static constexpr int BAR_BYTES = 256;
  static constexpr size_t SMEM = 1024 + static_cast<size_t>(STAGES) * STAGE_BYTES + BAR_BYTES;
  static_assert((2 * STAGES + 5) * 8 + 8 <= BAR_BYTES, "barrier area");
  static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM allocation");
  static_assert(STAGE_BYTES % 1024 == 0 && A_BYTES % 1024 == 0, "swizzle atoms stay aligned");
};

struct Tile {
  int g, mt, nc, n_valid;
};

// Tile w -> (group, weight block, token block); tile_start is the exclusive
// prefix of per-group tile counts, so the group is the last g with
// tile_start[g] <= w (empty groups are skipped naturally).
__device__ __forceinline__ Tile decode_tile(const GemmParams& p, int w) {
  if (p.single_rows > 0) {
    Tile t;
    t.g = 0;
    t.nc = w / p.m_tiles;
    t.mt = w - t.nc * p.m_tiles;
    t.n_valid = min(kBN, p.single_rows - t.nc * kBN);
    return t;
  }
  int lo = 0, hi = p.G;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.tile_start[mid] <= w)
      lo = mid;
    else
      hi = mid;
  }
  Tile t;
  t.g = lo;
  const int local = w - p.tile_start[lo];
  t.nc = local / p.m_tiles;
  t.mt = local - t.nc * p.m_tiles;
  t.n_valid = min(kBN, p.counts[lo] - t.nc * kBN);
  return t;
}

__device__ __forceinline__ int total_tiles(const GemmParams& p) {
  if (p.single_rows > 0) return p.m_tiles * ((p.single_rows + kBN - 1) / kBN);
  return p.tile_start[p.G];
}

__device__ __forceinline__ int group_row0(const GemmParams& p, int g) {
  return p.single_rows > 0 ? 0 : p.row_start[g];
}

template <int MODE>
__global__ void __launch_bounds__(192, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmBsh, const GemmParams p) {
  using S = Shape<MODE>;
  constexpr bool GU = S::GU;
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
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    if (GU) prefetch_tmap(&tmBsh);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), S::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = total_tiles(p);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_a = l2_policy_evict_first();  // weights: streamed once
      const uint64_t pol_b = l2_policy_evict_last();   // token rows: reused by every weight block
      uint32_t it = 0;
      for (int w = blockIdx.x; w < total; w += gridDim.x) {
        if (*abort_flag) break;
        const Tile t = decode_tile(p, w);
        const int n_mma = (t.n_valid + 15) & ~15;
        const int nbox = (n_mma + kBBoxRows - 1) / kBBoxRows;
        const bool sh = GU && t.g == p.E;
        const CUtensorMap* mb = sh ? &tmBsh : &tmB;
        const int b_row = (sh ? p.shared_b_row0 : group_row0(p, t.g)) + t.nc * kBN;
        const int a_row = t.g * p.a_rows_per_group + t.mt * S::A_ROWS;
        const uint32_t bytes = S::A_BYTES + nbox * S::B_BOX_BYTES;
        bool ok = true;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          const uint32_t s = it % S::STAGES;
          const uint32_t ph = (it / S::STAGES) & 1u;
          if (!mbar_wait(empty0 + 8 * s, ph ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          const uint32_t fb = full0 + 8 * s;
          mbar_arrive_expect_tx(fb, bytes);
          const uint32_t sa = smem_u32(smem + s * S::STAGE_BYTES);
          const uint32_t sb = sa + S::A_BYTES;
          tma_load_2d(sa, &tmA, fb, kb * kBK, a_row, pol_a);
          const int bk = p.b_k_wrap > 0 ? (kb * kBK) % p.b_k_wrap : kb * kBK;
          for (int i = 0; i < nbox; ++i)
            tma_load_2d(sb + i * S::B_BOX_BYTES, mb, fb, bk, b_row + i * kBBoxRows, pol_b);
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
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tc = 0;
      for (int w = blockIdx.x; w < total; w += gridDim.x) {
        if (*abort_flag) break;
        const Tile t = decode_tile(p, w);
        const int n_mma = (t.n_valid + 15) & ~15;
        const uint32_t idesc = idesc_bf16_f32(kBM, n_mma);
        const uint32_t buf = tc & 1u;
        const uint32_t tph = (tc >> 1) & 1u;
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
          const uint32_t sa = smem_u32(smem + s * S::STAGE_BYTES);
          const uint32_t sb = sa + S::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t bdesc = sdesc_k_sw128(sb + kk * 32);
            const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
            tc_mma_bf16(d, sdesc_k_sw128(sa + kk * 32), bdesc, idesc, acc);
            if (GU) tc_mma_bf16(d + kBN, sdesc_k_sw128(sa + kBM * 128 + kk * 32), bdesc, idesc, acc);
          }
          tc_commit(empty0 + 8 * s);  // frees the stage once these MMAs have read it
          ++it;
        }
        if (!ok) break;
        tc_commit(tfull0 + 8 * buf);  // accumulator ready for the epilogue
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
    uint32_t tc = 0;
    for (int w = blockIdx.x; w < total; w += gridDim.x) {
      const Tile t = decode_tile(p, w);
      const uint32_t buf = tc & 1u;
      const uint32_t tph = (tc >> 1) & 1u;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(tfull0 + 8 * buf, tph, abort_flag, p.status) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * S::ACC_COLS;
      const int feat = t.mt * kBM + q * 32 + lane;
      const size_t row0 = static_cast<size_t>(group_row0(p, t.g)) + static_cast<size_t>(t.nc) * kBN;
      if (MODE == kModeRouter) {
        float* lp = p.out_f32 + row0 * p.out_ld + feat;
        const bool keep = feat < p.valid_feats;
        for (int c0 = 0; c0 < t.n_valid; c0 += 16) {
          uint32_t ra[16];
          tmem_ld_x16(taddr + c0, ra);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (keep && c0 + i < t.n_valid)
              lp[static_cast<size_t>(c0 + i) * p.out_ld] = __uint_as_float(ra[i]);
        }
      } else if (GU) {
        __nv_bfloat16* outp = p.out + row0 * p.out_ld + feat;
        const float L = (t.g == p.E) ? p.limit_shared : p.limit;
        for (int c0 = 0; c0 < t.n_valid; c0 += 16) {
          uint32_t ra[16], rb[16];
          tmem_ld_x16(taddr + c0, ra);
          tmem_ld_x16(taddr + kBN + c0, rb);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if (c0 + i < t.n_valid) {
              float a = __uint_as_float(ra[i]);
              float u = __uint_as_float(rb[i]);
              if (L > 0.f) {
                a = fminf(a, L);
                u = fminf(fmaxf(u, -L), L);
              }
              const float hv = a / (1.0f + __expf(-a)) * u;
              outp[static_cast<size_t>(c0 + i) * p.out_ld] = __float2bfloat16_rn(hv);
            }
          }
        }
      } else {
        __nv_bfloat16* outp = p.out + row0 * p.out_ld + feat;
        const float* wrow = p.w_perm + row0;
        for (int c0 = 0; c0 < t.n_valid; c0 += 16) {
          uint32_t ra[16];
          tmem_ld_x16(taddr + c0, ra);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if (c0 + i < t.n_valid) {
              const float yv = __uint_as_float(ra[i]) * wrow[c0 + i];
              outp[static_cast<size_t>(c0 + i) * p.out_ld] = __float2bfloat16_rn(yv);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * buf);
      ++tc;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, S::TMEM_COLS);
  }
}

}  // namespace

size_t gemm_smem_bytes(int mode) {
  return mode == kModeGateUp ? Shape<kModeGateUp>::SMEM
                             : (mode == kModeDown ? Shape<kModeDown>::SMEM : Shape<kModeRouter>::SMEM);
}

cudaError_t gemm_configure_device() {
  cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<kModeGateUp>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(Shape<kModeGateUp>::SMEM));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(grouped_gemm_kernel<kModeDown>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(Shape<kModeDown>::SMEM));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(grouped_gemm_kernel<kModeRouter>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(Shape<kModeRouter>::SMEM));
}

cudaError_t launch_gemm_gate_up(const CUtensorMap& tmA, const CUtensorMap& tmB,
                                const CUtensorMap& tmBsh, const GemmParams& p, int grid,
                                cudaStream_t st) {
  grouped_gemm_kernel<kModeGateUp><<<grid, 192, Shape<kModeGateUp>::SMEM, st>>>(tmA, tmB, tmBsh, p);
  return cudaGetLastError();
}

cudaError_t launch_gemm_down(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmParams& p,
                             int grid, cudaStream_t st) {
  grouped_gemm_kernel<kModeDown><<<grid, 192, Shape<kModeDown>::SMEM, st>>>(tmA, tmB, tmB, p);
  return cudaGetLastError();
}

cudaError_t launch_gemm_router(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmParams& p,
                               int grid, cudaStream_t st) {
  grouped_gemm_kernel<kModeRouter><<<grid, 192, Shape<kModeRouter>::SMEM, st>>>(tmA, tmB, tmB, p);
  return cudaGetLastError();
}

}  // namespace moe
