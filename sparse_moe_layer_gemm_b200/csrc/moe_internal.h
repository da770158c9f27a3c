// Internal interfaces between the C-ABI layer (moe_api.cu) and the kernel
// translation units.  Not installed, not part of the ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

// Tile shape of the grouped GEMMs (swap-AB: weight rows are the MMA's M side,
// the group's tokens its N side).
constexpr int kBM = 128;        // weight rows per MMA
constexpr int kBK = 64;         // K elements per pipeline stage (one 128-byte row)
constexpr int kBK32 = 32;       // the same for fp32 (tf32) operands
constexpr int kBN = 128;        // tokens per tile (MMA N is rounded up to 16)
constexpr int kBBoxRows = 32;   // token rows per TMA box of the B operand

// Router tile (SIMT fp32): tokens x experts per block.
constexpr int kRouterTok = 64;
constexpr int kRouterExp = 96;
constexpr int kRouterKStep = 32;

// Groups (routed experts + the shared one) the grouped GEMM supports.
constexpr int kMaxGroups = 1025;

// Chunk of tokens owned by one block of the counting sort (4 x 32-bit masks).
constexpr int kSortChunk = 128;

// Epilogue modes of the grouped GEMM kernel.
constexpr int kModeGateUp = 0;  // h = silu(clamp(gate)) * clamp(up), bf16
constexpr int kModeDown = 1;    // y = acc * w_perm[row], bf16
constexpr int kModeRouter = 2;  // logits = acc, fp32, features < valid_feats
constexpr int kModePartial = 3; // split-K part z of one group: raw fp32 accumulators of
                                // every packed weight row, at out_f32 + z * part_stride

// Token count from which the expert GEMMs run on CTA pairs (2-SM UMMA,
// 256-token tiles; needs an even number of 128-feature blocks in H).
constexpr int kPairMinTokens = 2048;

// FP8-weight expert GEMMs: tokens per tile (two buffers of up to four
// 128 x kFp8BN partial accumulators fill half of tensor memory; the expanded
// weight operands take the other half).
constexpr int kFp8BN = 32;

// Token count from which the router runs on the tensor cores (bf16 x only),
// and the K parts of its reduction (the three bf16 terms of W_r).
constexpr int kTcRouterMinTokens = 512;
constexpr int kRouterTcParts = 3;

struct GemmParams {
  int single_rows;        // > 0: one group of this many rows starting at row 0
                          // (counts / row_start / tile_start unused)
  const int* counts;      // [G] rows per group (group E = the shared expert, T rows)
  const int* row_start;   // [G + 1] first row of each group in x_perm / h / y
  const int* tile_start;  // [G + 1] exclusive prefix of the group's tile counts
  int G;                  // groups = E + 1
  int E;                  // routed experts (index of the shared group)
  int num_kb;             // K / kBK
  int m_tiles;            // weight-row tiles per group
  int a_rows_per_group;   // rows of the packed A operand per group
  int shared_b_row0;      // gate/up: first row of the shared group's B operand
  __nv_bfloat16* out;     // h [rows, out_ld] or y [rows, out_ld]
  int out_ld;
  int out_feats;          // output features (columns) that exist; larger ones are not stored
  const float* w_perm;    // down: gate weight of each row (1 for shared rows)
  const float* a_scale;   // FP8 weights: scale of each packed weight row (A is
                          // E4M3 codes); nullptr: A is bf16
  const uint8_t* a_codes; // FP8 weights: the blocked code layout (see pack.cu)
  float limit;            // gate/up clamp of routed experts (<= 0: none)
  float limit_shared;     // gate/up clamp of the shared expert
  int* status;            // device status word
  int k_parts;            // single_rows: > 1 splits K into this many parts of num_kb
                          // k-blocks (A's K offset z * num_kb * kBK, B's 0), each part
                          // stored at out_f32 + z * part_stride (router: W1 | W2 | W3)
  size_t part_stride;
  float* out_f32;         // router: logits [rows, out_ld]; fp32 expert path: h as
                          // [rows, out_ld] with out_ld = 2 * I_pad (tf32 hi | lo), or y
  int valid_feats;        // router: features (experts) actually stored
  int kb_term;            // fp32 expert path: k-blocks (kBK32) per term; A and B hold
                          // [hi | lo] halves of kb_term k-blocks each, and num_kb =
                          // 3 * kb_term walks the terms hi.hi, lo.hi, hi.lo
};

// Guard band (selection-score units) of the top-k after the tensor-core
// router: experts whose approximate score is within it of the approximate
// k-th are recomputed in fp32 on the CUDA cores.  Sized from a worst-case
// accumulation error: 3H/16 MMA steps, each truncating at most one fp32 ulp
// of partial sums up to magnitude 8 (2^-20), times the sigmoid's maximum
// slope 0.25, times 2 for the two sides of the boundary -- ~3.7e-4 at
// H = 4096, against ~2.8e-5 observed.
__host__ __device__ constexpr float router_refine_band(int H) {
  return 2.0f * 0.25f * (3.0f * H / 16.0f) * 9.5367431640625e-07f;
}

struct TopkRefine {
  const __nv_bfloat16* x;  // [T, H] bf16 input rows
  const float* w_t;        // [E, H] fp32 router weight, transposed
  int H;
  float band;              // 0: no refinement
};

// ---- launchers (each returns the cudaGetLastError of its launch) ----
cudaError_t launch_router_logits(const void* x, bool x_bf16, const float* router_w, float* partial,
                                 int T, int H, int E, int ksplit, cudaStream_t st);
cudaError_t launch_topk(const float* partial, int ksplit, int T, int E, int k, const float* bias,
                        bool norm, float scale, int* topk_idx, float* topk_w, cudaStream_t st,
                        float* logits_out = nullptr, const TopkRefine* refine = nullptr);
// shared_rows: T, or 0 for an expert shard without the shared expert; ids
// outside [0, E) are another shard's experts (pos -1)
cudaError_t launch_sort(const int* topk_idx, const float* topk_w, int T, int k, int E,
                        int shared_rows, int bn_gu, int bn_dn, int m_tiles_gu, int m_tiles_dn,
                        uint32_t* masks, int* chunk_cnt, int* chunk_base, int* counts,
                        int* row_start, int* tiles_gu, int* tiles_dn, int* perm, int* pos,
                        float* w_perm, cudaStream_t st);
// expert shard: local_idx = topk_idx - first inside [first, first + count), else -1
cudaError_t launch_localize(const int* topk_idx, int n, int first, int count, int* local_idx,
                            cudaStream_t st);
// x_perm rows: bf16 x by bulk copies per token (pos), else row by row (perm)
cudaError_t launch_gather(const void* x, bool x_bf16, const int* perm, const int* pos,
                          int rows_routed, int k, int T, int H, bool write_shared,
                          __nv_bfloat16* x_perm, int num_sms, int* status, cudaStream_t st);
// fp32 expert path: x_perm rows as [x_hi | x_lo] fp32 (2H per row, the tf32
// split), the routed rows (perm) then the shared expert's T rows
cudaError_t launch_gather_split(const void* x, bool x_bf16, const int* perm, int rows_routed,
                                int k, int T, int H, float* x_perm, int num_sms,
                                cudaStream_t st);
// 128-feature weight blocks per down-projection tile for hidden size H.
int gemm_down_blocks(int H);

// Tensor maps of one grouped-GEMM launch: the weight operand, the token-row
// operand with kBBoxRows- and BN-row boxes, the shared expert's token rows
// (gate|up only) with both box heights, and the output for TMA stores (h or
// y with 32-feature x 16-row boxes, no swizzle).  The CTA-pair kernels take
// a (wide stages) and a2 (narrow stages) for the weights and K-block maps for
// the token rows (see launch_gemm_gate_up_pair).
struct GemmMaps {
  CUtensorMap a, a2, b, bsh, bw, bshw, out;
};

cudaError_t launch_gemm_gate_up(const GemmMaps& m, const GemmParams& p, int grid, cudaStream_t st);
cudaError_t launch_gemm_down(const GemmMaps& m, const GemmParams& p, int grid, int blocks,
                             cudaStream_t st);
cudaError_t launch_gemm_router(const GemmMaps& m, const GemmParams& p, int grid, cudaStream_t st);
// fp32 expert path (kind::tf32, the three-term split; see tf32.cuh): m.a the
// [hi | lo] packed weights (fp32, 32-column x A-rows boxes), m.b / m.bw the
// [hi | lo] token rows (x_perm, the shared rows included, or h) with 32- and
// 128-row boxes; num_kb = 3 * kb_term; outputs through p.out_f32 (gate|up: h
// hi and lo halves, out_ld = 2 * I_pad; down: y fp32, out_ld = H).  m.out is
// not read.
cudaError_t launch_gemm_gate_up_tf32(const GemmMaps& m, const GemmParams& p, int grid,
                                     cudaStream_t st);
cudaError_t launch_gemm_down_tf32(const GemmMaps& m, const GemmParams& p, int grid, int blocks,
                                  cudaStream_t st);
// Split-K partial products of one group (single_rows, k_parts parts of num_kb
// k-blocks; A and B both offset by the part's K): m.a with 128-row boxes, two
// 128-row weight blocks per tile; fp32 [T, out_ld] per part.
cudaError_t launch_gemm_partial(const GemmMaps& m, const GemmParams& p, int grid, cudaStream_t st);
// CTA-pair versions (grouped_gemm_pair.cu), tiles of 256 tokens: m.a / m.a2
// the weights of wide / narrow stages (gate|up: encode_bf16_gate_up_pair with
// 2 / 3 K blocks; down: encode_bf16_kblocks, 128 rows, 2 / 3 K blocks); m.bw /
// m.bshw the token rows with 128-row x 2 K-block boxes, m.b / m.bsh with
// 32-row x 3 K-block boxes; num_kb = K / 64; m_tiles = I_pad / 128 (gate|up)
// or H / 256 (down).
cudaError_t launch_gemm_gate_up_pair(const GemmMaps& m, const GemmParams& p, cudaStream_t st);
cudaError_t launch_gemm_down_pair(const GemmMaps& m, const GemmParams& p, cudaStream_t st);
// FP8 E4M3 weights (grouped_gemm_fp8.cu): p.a_codes the tile-major code
// layout (tiles of 256 rows for gate|up, 128 * gemm_down_blocks(H) for down;
// see pack.cu), p.a_scale the packed rows' scales; m.b / m.bsh the token rows
// as 3-D maps (64 columns x kFp8BN rows x 2 K-blocks boxes, see
// encode_bf16_kpair); one-SM tiles of kFp8BN tokens at every T.
cudaError_t launch_gemm_gate_up_fp8(const GemmMaps& m, const GemmParams& p, int grid,
                                    cudaStream_t st);
cudaError_t launch_gemm_down_fp8(const GemmMaps& m, const GemmParams& p, int grid, int blocks,
                                 cudaStream_t st);
cudaError_t launch_pack_router(const float* w, int H, int E, int E_pad, __nv_bfloat16* dst,
                               float* dst_t, cudaStream_t st);
cudaError_t launch_combine(const __nv_bfloat16* y, const int* pos, int T, int k, int H, bool out_bf16,
                           bool with_shared, void* out, cudaStream_t st);
// the same over fp32 rows y (the fp32 expert path)
cudaError_t launch_combine_f32(const float* y, const int* pos, int T, int k, int H, bool out_bf16,
                               bool with_shared, void* out, cudaStream_t st);
cudaError_t launch_pack_gate_up(const void* w, bool w_bf16, int groups, int H, int I, int I_pad,
                                int half, __nv_bfloat16* dst, cudaStream_t st);
cudaError_t launch_pack_down(const void* w, bool w_bf16, int groups, int H, int I, int I_pad,
                             __nv_bfloat16* dst, cudaStream_t st);
// fp32 expert path: the same rows, each as [hi | lo] fp32 halves of the tf32
// split (row length 2H for gate|up, 2 I_pad for down)
cudaError_t launch_pack_gate_up_split(const void* w, bool w_bf16, int groups, int H, int I,
                                      int I_pad, int half, float* dst, cudaStream_t st);
cudaError_t launch_pack_down_split(const void* w, bool w_bf16, int groups, int H, int I,
                                   int I_pad, float* dst, cudaStream_t st);
// FP8 E4M3 weights: the same packing, one byte per code, and the gate|up
// rows' scales (down's scales need no reordering: row g * H + n)
cudaError_t launch_pack_codes_gate_up(const uint8_t* w, int groups, int H, int I, int I_pad,
                                      int half, uint8_t* dst, cudaStream_t st);
cudaError_t launch_pack_codes_down(const uint8_t* w, int groups, int H, int I, int I_pad,
                                   int tile_rows, uint8_t* dst, cudaStream_t st);
cudaError_t launch_pack_gate_up_scales(const float* s, int groups, int I, int I_pad, int half,
                                       float* dst, cudaStream_t st);
// n E4M3 codes (n % 4 == 0, 4-byte aligned) -> n bf16 values
cudaError_t launch_decode_e4m3(const uint8_t* codes, size_t n, __nv_bfloat16* out,
                               cudaStream_t st);

// The fused persistent forward (fused_moe.cu): bf16 x and weights, from
// kPairMinTokens tokens, H / 128 even, E <= kFusedMaxExperts (the top-k's
// experts per lane, kFusedMPL, is fixed).
constexpr int kFusedMaxExperts = 288;
constexpr int kFusedMPL = 9;
// K parts of the fused kernel's tensor-core router: each bf16 term's K in two
// halves (partial logits [kFusedRouterParts, T, E])
constexpr int kFusedRouterParts = 6;

struct FusedLaunch {
  // tensor maps: weights of wide / narrow stages (router: encode_bf16_kblocks
  // of the packed three-term split, 128 rows; gate|up: encode_bf16_gate_up_pair;
  // down: encode_bf16_kblocks, 128 rows), token rows of x and h (128 rows x 2
  // and 32 rows x 3 K blocks), and the TMA stores of h and y
  CUtensorMap rt_w, rt_n, gu_w, gu_n, dn_w, dn_n, x_w, x_n, h_w, h_n, st_h, st_y;
  CUtensorMap xp_w, xp_n;  // x_perm's K-block maps (gather phase only)
  __nv_bfloat16* x_perm;   // non-null: gather the routed rows in a phase of their own
  const __nv_bfloat16* x;
  __nv_bfloat16* out;
  int T, H, E, k, I_pad;
  const float* bias;      // [E] or nullptr
  const float* router_t;  // [E, H]
  float band;
  int norm;
  float scale;
  int rt_mtiles;          // ceil(E_pad / 256)
  float* logits_out;      // optional [T, E]
  float* partial;         // [kFusedRouterParts, T, E]
  int *topk_idx;
  float* topk_w;
  uint32_t* masks;
  int *chunk_cnt, *chunk_base, *counts, *row_start, *tiles_gu, *tiles_dn, *perm, *pos;
  float* w_perm;
  __nv_bfloat16 *h, *y;
  unsigned int* sync;     // zeroed before the launch: [0] grid barrier, [1 + b] token block b
  float limit, limit_shared;
  int* status;
  uint64_t wait_ns;       // limit of every bounded wait (0: the default, 2 s)
  unsigned int ready_extra;  // self-check only: unreachable readiness target (0 in a forward)
};

// Readiness counters of the fused forward for T tokens and G groups: one per
// 256-token block of every group's rows, plus the grid barrier's.
inline size_t fused_sync_words(int T, int k, int G) {
  return 1 + static_cast<size_t>(T) * (k + 1) / 256 + static_cast<size_t>(G) + 1;
}

cudaError_t fused_configure_device(int num_sms);
cudaError_t launch_fused(const FusedLaunch& f, cudaStream_t st);

// Launches `kernel` on `st` with programmatic stream serialization, so it may
// start (up to its pdl_wait) while the previous kernel of the stream ends.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// one-time per-device kernel attribute setup (dynamic shared memory limits)
cudaError_t gemm_configure_device();
cudaError_t gemm_fp8_configure_device();
// also sizes the pair kernels' grid to the co-resident 2-CTA clusters
cudaError_t gemm_pair_configure_device(int num_sms);
cudaError_t topk_configure_device();
cudaError_t gather_configure_device();


}  // namespace moe
