// Host-side helpers shared by the C-ABI translation units (moe_api.cu,
// dense_api.cu): tensor-map encoders, the device guard, argument checks.
// Not installed, not part of the ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// bf16 [rows, cols] row-major, box = 64 columns (128 bytes) x box_rows, 128B
// swizzle; out-of-range elements read as zero.
bool encode_bf16_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                    uint32_t box_rows);
// fp32 [rows, cols] row-major, box = 32 columns (128 bytes) x box_rows, 128B
// swizzle (the fp32 path's tf32 operands); out-of-range elements read as zero.
bool encode_f32_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                   uint32_t box_rows);
// bf16 [rows, cols] as 3-D (64 columns, rows, cols / 64 column blocks), box
// 64 x box_rows x kblocks column blocks, 128B swizzle: in shared memory the
// box is k-block-major (kblocks sub-blocks of box_rows 128-byte rows).
bool encode_bf16_kblocks(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                         uint32_t box_rows, uint32_t kblocks);
inline bool encode_bf16_kpair(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                              uint32_t box_rows) {
  return encode_bf16_kblocks(m, base, rows, cols, box_rows, 2);
}
// The packed gate|up weights [rows, cols] (blocks of 128 gate rows then 128
// up rows) as 4-D (64 columns, rows - 128, 2 halves 128 rows apart, cols / 64
// column blocks), box 64 x 64 rows x 2 halves x kblocks, 128B swizzle: one
// CTA of a pair gets its 64 gate rows and the matching 64 up rows of every
// K sub-block of a stage in one load; in shared memory per sub-block the 64
// gate rows, then the 64 up rows.  (The row extent stops 128 short of the
// tensor, so every element the map can address lies inside it.)
bool encode_bf16_gate_up_pair(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                              uint32_t kblocks);
// bf16 [rows, cols] row-major, box 32 columns x 16 rows, no swizzle (the GEMM
// epilogues' TMA stores).
bool encode_bf16_store(CUtensorMap* m, void* base, uint64_t rows, uint64_t cols);

inline bool aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

// Makes a device current for the lifetime of the guard.
struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) {
      ok = false;
      return;
    }
    if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

}  // namespace moe

#define MOE_CUDA(call)                              \
  do {                                              \
    if ((call) != cudaSuccess) return MOE_ERR_CUDA; \
  } while (0)
