// Shared definitions of the GDN kernels: status word, problem description, smem layout
// constants.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace gdn {

// Device status word: 0 = OK, otherwise the first error a kernel recorded (the C-ABI status
// codes; GDN_ERR_TIMEOUT when a bounded wait ran out). Read and cleared by gdn_sync_status.
__device__ int g_status;

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_status, 0, code); }

constexpr int kErrTimeout = 6;  // == GDN_ERR_TIMEOUT

// One problem: q/k/v/out are [B, T, N, H, D] bf16, gamma/beta [B, T, H] f32.
struct Problem {
  int B, H, T, N, D;
  float key_scale;
};

// TMA box: 64 bf16 (128 B, one swizzle row) x 128 rows.
constexpr int kRowsPerTile = 128;
constexpr int kBoxBytes = 128 * 128;  // 16 KB

// Round an address up to 1 KB (swizzle-atom alignment of every tile).
__device__ __forceinline__ uint8_t* align1k(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

}  // namespace gdn
