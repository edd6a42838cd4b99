// Block-causal linear attention state: the state is additive (the state of block i is the
// cached state of block i-1 plus block i's own contribution), so the scan over frames is a
// running sum of the per-block statistics [V | 1]^T relu(K) (each block's frames already summed
// by the statistics kernel). One thread owns one element of the augmented (D+1) x D matrix of
// one head (row D = normaliser z) and walks the blocks, writing the bf16 state after every block
// for the output GEMM. Coalesced over elements; HBM-bound on reading the block sums once.
//
// External state layout (as the block-causal formulation writes it): S [B, H, D_k, D_v] f32,
// z [B, H, D_k] f32. Internal layout: row v (value; v == D is z), column k (key).
#pragma once
#include "common.cuh"

namespace gdn {

// B_ws / S_ws rows: (b*H + h)*n_blocks + block, each (D+1) x D (per-block sums / states).
__global__ void __launch_bounds__(256)
    gdn_la_scan_kernel(const float* __restrict__ B_ws, __nv_bfloat16* __restrict__ S_ws,
                       const float* __restrict__ state_in, const float* __restrict__ z_in,
                       float* __restrict__ state_out, float* __restrict__ z_out, int n_blocks,
                       int D) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;  // element of the (D+1) x D matrix
  const int per = (D + 1) * D;
  if (e >= per) return;
  const int v = e / D;
  const int k = e - v * D;
  float acc = 0.f;
  if (v < D) {
    if (state_in) acc = state_in[(static_cast<long>(bh) * D + k) * D + v];
  } else {
    if (z_in) acc = z_in[static_cast<long>(bh) * D + k];
  }
  const long base = static_cast<long>(bh) * n_blocks;
  int j = 0;
  for (; j + 4 <= n_blocks; j += 4) {  // four independent loads in flight
    float x[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) x[u] = __ldg(B_ws + (base + j + u) * per + e);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      acc += x[u];
      S_ws[(base + j + u) * per + e] = __float2bfloat16(acc);
    }
  }
  for (; j < n_blocks; ++j) {
    acc += __ldg(B_ws + (base + j) * per + e);
    S_ws[(base + j) * per + e] = __float2bfloat16(acc);
  }
  if (v < D) {
    if (state_out) state_out[(static_cast<long>(bh) * D + k) * D + v] = acc;
  } else {
    if (z_out) z_out[static_cast<long>(bh) * D + k] = acc;
  }
}

}  // namespace gdn
