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
constexpr int kBN = 128;        // tokens per tile (MMA N is rounded up to 16)
constexpr int kBBoxRows = 32;   // token rows per TMA box of the B operand

// Router tile (SIMT fp32): tokens x experts per block.
constexpr int kRouterTok = 64;
constexpr int kRouterExp = 96;
constexpr int kRouterKStep = 32;

// Chunk of tokens owned by one block of the counting sort (4 x 32-bit masks).
constexpr int kSortChunk = 128;

struct GemmParams {
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
  const float* w_perm;    // down: gate weight of each row (1 for shared rows)
  float limit;            // gate/up clamp of routed experts (<= 0: none)
  float limit_shared;     // gate/up clamp of the shared expert
  int* status;            // device status word
};

// ---- launchers (each returns the cudaGetLastError of its launch) ----
cudaError_t launch_router_logits(const void* x, bool x_bf16, const float* router_w, float* partial,
                                 int T, int H, int E, int ksplit, cudaStream_t st);
cudaError_t launch_topk(const float* partial, int ksplit, int T, int E, int k, const float* bias,
                        bool norm, float scale, int* topk_idx, float* topk_w, cudaStream_t st);
cudaError_t launch_sort(const int* topk_idx, const float* topk_w, int T, int k, int E, int m_tiles_gu,
                        int m_tiles_dn, uint32_t* masks, int* chunk_cnt, int* chunk_base,
                        int* counts, int* row_start, int* tiles_gu, int* tiles_dn, int* perm,
                        int* pos, float* w_perm, cudaStream_t st);
cudaError_t launch_gather(const void* x, bool x_bf16, const int* perm, int rows_routed, int k, int T,
                          int H, bool write_shared, __nv_bfloat16* x_perm, int num_sms,
                          cudaStream_t st);
cudaError_t launch_gemm_gate_up(const CUtensorMap& tmA, const CUtensorMap& tmB,
                                const CUtensorMap& tmBsh, const GemmParams& p, int grid,
                                cudaStream_t st);
cudaError_t launch_gemm_down(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmParams& p,
                             int grid, cudaStream_t st);
cudaError_t launch_combine(const __nv_bfloat16* y, const int* pos, int T, int k, int H, bool out_bf16,
                           void* out, cudaStream_t st);
cudaError_t launch_pack_gate_up(const void* w, bool w_bf16, int groups, int H, int I, int I_pad,
                                int half, __nv_bfloat16* dst, cudaStream_t st);
cudaError_t launch_pack_down(const void* w, bool w_bf16, int groups, int H, int I, int I_pad,
                             __nv_bfloat16* dst, cudaStream_t st);

// one-time per-device kernel attribute setup (dynamic shared memory limits)
cudaError_t gemm_configure_device();
size_t gemm_smem_bytes(bool gate_up);

}  // namespace moe
