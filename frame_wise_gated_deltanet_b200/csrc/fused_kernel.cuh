// Fused forward: one persistent, co-resident grid (cooperative launch, one CTA per SM) runs
// the three stages concurrently so that the serial state chain overlaps the two HBM streams.
//
//   blocks [0, B*H)              chain role, one per (batch, head)
//   blocks [B*H, B*H + n_stats)  stats role: A_t, B_t of frame-major items into ring slots
//   blocks [.., gridDim.x)       output role: O_t from ring slots of S_t
//
// A_t (bf16), B_t (f32) and S_t (bf16) travel through per-head rings of R slots (a few tens of
// MB, meant to stay in L2: A_t and S_t are loaded with evict_last while the q/k/v/out streams
// use evict_first). Hand-off is by release/acquire flags in global memory with bounded waits;
// the statistics take items in frame-major order and the outputs in the order the chains
// publish them (frame order within a head); every wait points at a strictly earlier frame, at
// the chain (which only waits on earlier frames) or at a queue position the chains will fill, so
// with all CTAs co-resident the grid cannot deadlock.
#pragma once
#include <cuda.h>

#include "chain_kernel.cuh"
#include "common.cuh"
#include "output_kernel.cuh"
#include "stats_kernel.cuh"

namespace gdn {

constexpr int cmax(int a, int b) { return a > b ? a : b; }

// Epilogue warp groups of the output role (see output_kernel.cuh). DP = 128: one group (with
// four the 720p clip ran 16 % slower although the standalone output kernel gains from them).
// DP = 64: two, so that the role's read-out keeps pace with the chain's short frame steps.
#ifndef GDN_FUSED_OUT_GROUPS
#define GDN_FUSED_OUT_GROUPS 1
#endif
#ifndef GDN_FUSED_OUT_GROUPS_64
#define GDN_FUSED_OUT_GROUPS_64 2
#endif
template <int DP>
constexpr int kFusedOutGroups = DP == 64 ? GDN_FUSED_OUT_GROUPS_64 : GDN_FUSED_OUT_GROUPS;

// Groups of 128 threads in the RoPE transform of the statistics and output roles: three at
// DP = 128 (12 warps; the 720p clip measured 4.90 ms against 5.25 with two), two at DP = 64
// (whose output role has two epilogue groups, so 12 transform warps would not fit its 19).
#ifndef GDN_FUSED_ROPE_GROUPS
#define GDN_FUSED_ROPE_GROUPS 3
#endif
template <int DP>
constexpr int kFusedRopeGroups = DP == 128 ? GDN_FUSED_ROPE_GROUPS : 2;

template <int DP>
struct FusedLayout {
  static constexpr int kThreads = ChainLayout<DP>::kThreads;
  static_assert(kThreads >= StatsLayout<DP, false, DP == 128>::kThreads &&
                    kThreads >= OutputLayout<DP, false, kFusedOutGroups<DP>, DP == 128>::kThreads &&
                    kThreads >= StatsLayout<DP, false, false, true, kFusedRopeGroups<DP>>::kThreads &&
                    kThreads >= OutputLayout<DP, false, kFusedOutGroups<DP>, false, true,
                                             kFusedRopeGroups<DP>>::kThreads,
                "the chain role's CTA size must cover the other roles' warps");
  // the statistics role's publisher is the CTA's last warp (warp 18), past its transform warps
  static_assert(kThreads / 32 - 1 == 18 &&
                    6 + StatsLayout<DP, false, DP == 128>::kTransformThreads / 32 <= 18 &&
                    6 + StatsLayout<DP, false, false, true, kFusedRopeGroups<DP>>::kTransformThreads /
                            32 <= 18,
                "statistics publisher warp");
  static_assert(2 + 4 * kFusedOutGroups<DP> +
                        OutputLayout<DP, false, kFusedOutGroups<DP>, DP == 128>::kXfWarps <= 18 &&
                    2 + 4 * kFusedOutGroups<DP> +
                            OutputLayout<DP, false, kFusedOutGroups<DP>, false, true,
                                         kFusedRopeGroups<DP>>::kXfWarps <= 18,
                "output publisher warp");
  static constexpr int kSmemBytes = cmax(
      cmax(ChainLayout<DP>::kSmemBytes,
           cmax(StatsLayout<DP, false>::kSmemBytes, OutputLayout<DP, false>::kSmemBytes)),
      cmax(StatsLayout<DP, false, DP == 128>::kSmemBytes,
           OutputLayout<DP, false, kFusedOutGroups<DP>, DP == 128>::kSmemBytes));
  // with RoPE the statistics and output roles also hold the table copy of rope_stage_rc
  static constexpr int kSmemBytesRope =
      cmax(kSmemBytes, cmax(StatsLayout<DP, false, false, true, kFusedRopeGroups<DP>>::kSmemBytes,
                            OutputLayout<DP, false, kFusedOutGroups<DP>, false, true,
                                         kFusedRopeGroups<DP>>::kSmemBytes));
};

// kF8: e4m3 q, k, v with per (b, t, h) scales in p (DP = 128 only). kRope: q and k rotated by
// the 3D RoPE of p.rope in shared memory by the statistics and output roles.
template <int DP, bool kF8 = false, bool kRope = false>
__global__ void __launch_bounds__(FusedLayout<DP>::kThreads, 1)
    gdn_fused_kernel(const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_o,
                     const __grid_constant__ CUtensorMap tm_a_ring,
                     __nv_bfloat16* __restrict__ A_ring, float* __restrict__ B_ring,
                     __nv_bfloat16* __restrict__ S_ring,
                     const float* __restrict__ gamma, const float* __restrict__ beta,
                     const float* __restrict__ state_in, float* __restrict__ state_out, Problem p,
                     Handoff h_chain, Handoff h_stats, Handoff h_out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1k(smem_raw);
  if (static_cast<int>(blockIdx.x) < h_stats.base) {
    const ChainSeg whole{p.T, 1, 0, nullptr, nullptr};
    chain_body<DP, true>(&tm_a_ring, B_ring, S_ring, gamma, beta, state_in, state_out, p,
                         h_chain, whole, smem);
  } else if (static_cast<int>(blockIdx.x) < h_out.base) {
    stats_body<DP, false, true, true, kF8, kRope, kFusedRopeGroups<DP>>(&tm_k, &tm_v, A_ring,
                                                                       B_ring, p, h_stats, smem);
  } else {
    output_body<DP, false, true, kFusedOutGroups<DP>, kF8, kRope, kFusedRopeGroups<DP>>(
        &tm_q, &tm_q, S_ring, &tm_o, p, 1, h_out, smem);
  }
}

}  // namespace gdn
