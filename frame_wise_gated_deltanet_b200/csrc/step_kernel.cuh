// Fused single-frame streaming step: for every (batch, head), in one pass and one launch,
//
//   A = s^2 K^T K,  B = s V^T K        (tcgen05, K and V tiles MN-major from TMA)
//   P = S_in A                          (tcgen05, S_in and A as bf16 core-matrix tiles)
//   S_out = gamma (S_in - beta P) + beta B   (fp32, identity part exact)
//   O = Q S_out^T                       (tcgen05, S_out as the bf16 B operand)
//
// so nothing goes through global memory but the inputs, the state and the output. The CTA is
// persistent over (batch, head) items; while the epilogue finishes one item's output tiles the
// MMA warp already accumulates the next item's statistics.
//
// Shared memory: a ring of 32 KB stages, each one 128-token x 128-dim bf16 tile (K, V and Q
// tiles stream through the same ring), the S tile (state, then updated state, as 8-row x 16 B
// core matrices) and the X tile (A as core matrices, then the bf16 output staging for the TMA
// stores). TMEM: columns [0,128) A then P, [128,256) B, [256,512) two output accumulators.
//
// Warps: 0 TMA producer, 1 TMEM allocator + MMA issuer, 2..9 epilogue (warp w: rows
// 32*(w%4).., column half (w-2)/4).
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace gdn {

struct StepLayout {
  static constexpr int kStageBytes = 2 * kBoxBytes;  // 128 x 128 bf16 tile (two TMA boxes)
  static constexpr int kStages = 5;
  static constexpr int kTileBytes = 128 * 128 * 2;   // S and X tiles
  static constexpr int kThreads = 320;
  static constexpr int kTmemCols = 512;
  static constexpr int kSmemBytes = kStages * kStageBytes + 2 * kTileBytes + 512 + 1024;
};

// q, k, v, out tensor maps over [B, 1, N, H, D] (T = 1); gamma, beta [B, H]; state [B, H, D, D].
__global__ void __launch_bounds__(StepLayout::kThreads, 1)
    gdn_step_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_o, const float* __restrict__ gamma,
                    const float* __restrict__ beta, const float* state_in, float* state_out,
                    Problem p) {
  using L = StepLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1k(smem_raw);
  uint8_t* s_tile = smem + L::kStages * L::kStageBytes;
  uint8_t* x_tile = s_tile + L::kTileBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(x_tile + L::kTileBytes);
  uint64_t* empty = full + L::kStages;
  uint64_t* stats_done = empty + L::kStages;  // A, B accumulated
  uint64_t* sa_ready = stats_done + 1;        // S tile and A tile written
  uint64_t* p_done = sa_ready + 1;            // P = S A accumulated
  uint64_t* s2_ready = p_done + 1;            // updated state in the S tile; P, B read
  uint64_t* s_free = s2_ready + 1;            // the item's output MMAs are done with the S tile
  uint64_t* o_full = s_free + 1;              // [2]
  uint64_t* o_empty = o_full + 2;             // [2]
  uint64_t* mma_drain = o_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const long n_items = static_cast<long>(p.B) * p.H;
  const int n_tiles = (p.N + kRowsPerTile - 1) / kRowsPerTile;
  const int D = p.D;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(stats_done, 1);
    mbar_init(sa_ready, 256);
    mbar_init(p_done, 1);
    mbar_init(s2_ready, 256);
    mbar_init(s_free, 1);
    for (int a = 0; a < 2; ++a) {
      mbar_init(&o_full[a], 1);
      mbar_init(&o_empty[a], 256);
    }
    mbar_init(mma_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (elect_one()) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const uint64_t pol = policy_evict_first();
      StageFills<L::kStages> fills;
      int stage = 0;
      uint32_t phase = 0;
      auto load_tile = [&](const CUtensorMap* tm, int h, int tile, int b) -> bool {
        if (!mbar_wait(&empty[stage], phase ^ 1)) return false;
        mbar_arrive_expect_tx(&full[stage], L::kStageBytes);
        uint8_t* st = smem + stage * L::kStageBytes;
        tma_load_4d(st, tm, &full[stage], 0, h, tile * kRowsPerTile, b, pol);
        tma_load_4d(st + kBoxBytes, tm, &full[stage], 64, h, tile * kRowsPerTile, b, pol);
        fills.filled(stage, phase);
        if (++stage == L::kStages) {
          stage = 0;
          phase ^= 1;
        }
        return true;
      };
      bool ok = true;
      for (long item = blockIdx.x; item < n_items && ok && !*abort_flag; item += gridDim.x) {
        const int h = static_cast<int>(item % p.H);
        const int b = static_cast<int>(item / p.H);
        for (int tile = 0; tile < n_tiles && ok; ++tile)
          ok = load_tile(&tm_k, h, tile, b) && load_tile(&tm_v, h, tile, b);
        for (int tile = 0; tile < n_tiles && ok; ++tile) ok = load_tile(&tm_q, h, tile, b);
      }
      if (!ok) {
        record_error(kErrTimeout);
        *abort_flag = 1;
      }
      fills.drain(full);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc_stats = idesc_bf16(128, 128, true, true);
    constexpr uint32_t idesc_kmaj = idesc_bf16(128, 128, false, false);
    const uint32_t s_base = smem_u32(s_tile);
    const uint32_t x_base = smem_u32(x_tile);
    const uint32_t t_a = tmem_base, t_b = tmem_base + 128, t_o = tmem_base + 256;
    int stage = 0;
    uint32_t phase = 0;
    int tc = 0;
    bool ok = true;
    auto next_stage = [&]() {
      if (++stage == L::kStages) {
        stage = 0;
        phase ^= 1;
      }
    };
    int li = 0;
    for (long item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++li) {
      // the previous item's epilogue has read P and B (s2_ready), so A and B may be rewritten
      if (li > 0 && !mbar_wait(s2_ready, (li - 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int tile = 0; tile < n_tiles && ok; ++tile) {
        const int ks_stage = stage;
        if (!mbar_wait(&full[ks_stage], phase)) {
          ok = false;
          break;
        }
        next_stage();
        const int vs_stage = stage;
        if (!mbar_wait(&full[vs_stage], phase)) {
          ok = false;
          break;
        }
        next_stage();
        tc_fence_after();
        if (elect_one()) {
          const uint32_t kb = smem_u32(smem + ks_stage * L::kStageBytes);
          const uint32_t vb = smem_u32(smem + vs_stage * L::kStageBytes);
#pragma unroll
          for (int ks = 0; ks < kRowsPerTile / 16; ++ks) {
            const uint32_t accum = (tile | ks) != 0;
            const uint64_t dk = smem_desc(kb + ks * 2048, kBoxBytes, 1024);
            const uint64_t dv = smem_desc(vb + ks * 2048, kBoxBytes, 1024);
            mma_bf16(t_a, dk, dk, idesc_stats, accum);  // K^T K
            mma_bf16(t_b, dv, dk, idesc_stats, accum);  // V^T K
          }
          mma_commit(&empty[ks_stage]);
          mma_commit(&empty[vs_stage]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (elect_one()) mma_commit(stats_done);
      __syncwarp();
      // P = S_in A (into A's columns, which the epilogue has copied out)
      if (!mbar_wait(sa_ready, li & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t da = smem_desc_noswz(s_base + ks * 2 * 2048, 2048, 128);
          const uint64_t db = smem_desc_noswz(x_base + ks * 2 * 2048, 2048, 128);
          mma_bf16(t_a, da, db, idesc_kmaj, ks != 0);
        }
        mma_commit(p_done);
      }
      __syncwarp();
      // O = Q S_out^T, tile by tile
      if (!mbar_wait(s2_ready, li & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      for (int tile = 0; tile < n_tiles; ++tile, ++tc) {
        const int acc = tc & 1;
        if (!mbar_wait(&o_empty[acc], ((tc >> 1) & 1) ^ 1) || !mbar_wait(&full[stage], phase)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const uint32_t qb = smem_u32(smem + stage * L::kStageBytes);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            const uint64_t da = smem_desc(qb + (ks >> 2) * kBoxBytes + (ks & 3) * 32, 16, 1024);
            const uint64_t db = smem_desc_noswz(s_base + ks * 2 * 2048, 2048, 128);
            mma_bf16(t_o + acc * 128, da, db, idesc_kmaj, ks != 0);
          }
          mma_commit(&empty[stage]);
          mma_commit(&o_full[acc]);
        }
        __syncwarp();
        next_stage();
      }
      if (!ok) break;
      if (elect_one()) mma_commit(s_free);
      __syncwarp();
    }
    if (!ok) {
      record_error(kErrTimeout);
      *abort_flag = 1;
    }
    if (elect_one()) mma_commit(mma_drain);
    __syncwarp();
    mbar_wait(mma_drain, 0);
  } else {
    // ---------------------------------------------------------------- epilogue (256 threads)
    const uint32_t quarter = warp & 3;
    const int hf = (warp - 2) >> 2;
    const int v = quarter * 32 + lane;  // row: value index of S, key index k' of A
    const int c0 = hf * 64;             // first column owned
    const uint32_t lane_base = tmem_base + ((quarter * 32) << 16);
    const bool row_ok = v < D;
    const bool leader = (threadIdx.x == 64);
    const float s = p.key_scale;
    const float s2 = s * s;
    const uint64_t pol_out = policy_evict_first();
    if (leader) tma_prefetch_desc(&tm_o);
    auto core_off = [&](int col) { return (col >> 3) * 2048 + v * 16; };  // 8-column group
    int tc = 0;
    int li = 0;
    bool ok = true;
    for (long item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++li) {
      const int h = static_cast<int>(item % p.H);
      const int b = static_cast<int>(item / p.H);
      const long bh = item;
      const float g = __ldg(gamma + bh);
      const float be = __ldg(beta + bh);
      // S_in row v, this thread's 64 columns (fp32, kept for the update)
      float S[64];
      const float* sin = state_in ? state_in + (bh * D + v) * D : nullptr;
#pragma unroll
      for (int j = 0; j < 64; j += 4) {
        const int col = c0 + j;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (sin != nullptr && row_ok && col < D) x = *reinterpret_cast<const float4*>(sin + col);
        S[j] = x.x;
        S[j + 1] = x.y;
        S[j + 2] = x.z;
        S[j + 3] = x.w;
      }
      // the S tile and the X tile are free once the previous item's output MMAs are done and
      // its last output tile has been read out of the staging buffer
      bool bad = !mbar_wait(stats_done, li & 1) || (li > 0 && !mbar_wait(s_free, (li - 1) & 1));
      if (leader) bulk_wait_read<0>();
      if (named_bar_any(1, 256, bad)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int j = 0; j < 64; j += 8) {
        uint4 pk;
        pk.x = pack_bf16x2(S[j], S[j + 1]);
        pk.y = pack_bf16x2(S[j + 2], S[j + 3]);
        pk.z = pack_bf16x2(S[j + 4], S[j + 5]);
        pk.w = pack_bf16x2(S[j + 6], S[j + 7]);
        *reinterpret_cast<uint4*>(s_tile + core_off(c0 + j)) = pk;
      }
      // A row k' = v (A is symmetric), scaled, as a bf16 core-matrix operand
#pragma unroll 1
      for (int c = 0; c < 64; c += 32) {
        float a[32];
        tmem_ld32(lane_base + c0 + c, a);
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          uint4 pk;
          pk.x = pack_bf16x2(a[j] * s2, a[j + 1] * s2);
          pk.y = pack_bf16x2(a[j + 2] * s2, a[j + 3] * s2);
          pk.z = pack_bf16x2(a[j + 4] * s2, a[j + 5] * s2);
          pk.w = pack_bf16x2(a[j + 6] * s2, a[j + 7] * s2);
          *reinterpret_cast<uint4*>(x_tile + core_off(c0 + c + j)) = pk;
        }
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(sa_ready);
      // S_out = gamma (S_in - beta P) + beta s B
      if (named_bar_any(1, 256, !mbar_wait(p_done, li & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float gbe = g * be;
      const float bs = be * s;
#pragma unroll
      for (int c = 0; c < 64; c += 32) {
        float pp[32], bb[32];
        tmem_ld32(lane_base + c0 + c, pp);
        tmem_ld32(lane_base + 128 + c0 + c, bb);
#pragma unroll
        for (int j = 0; j < 32; ++j) S[c + j] = fmaf(g, S[c + j], fmaf(bs, bb[j], -gbe * pp[j]));
      }
      if (state_out != nullptr && row_ok) {
        float* so = state_out + (bh * D + v) * D;
#pragma unroll
        for (int j = 0; j < 64; j += 4)
          if (c0 + j < D)
            *reinterpret_cast<float4*>(so + c0 + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
      }
#pragma unroll
      for (int j = 0; j < 64; j += 8) {
        uint4 pk;
        pk.x = pack_bf16x2(S[j], S[j + 1]);
        pk.y = pack_bf16x2(S[j + 2], S[j + 3]);
        pk.z = pack_bf16x2(S[j + 4], S[j + 5]);
        pk.w = pack_bf16x2(S[j + 6], S[j + 7]);
        *reinterpret_cast<uint4*>(s_tile + core_off(c0 + j)) = pk;
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(s2_ready);
      // output tiles through the X tile as TMA-store staging (128B-swizzled, two boxes)
      for (int tile = 0; tile < n_tiles; ++tile, ++tc) {
        const int acc = tc & 1;
        const bool waited = mbar_wait(&o_full[acc], (tc >> 1) & 1);
        if (leader) bulk_wait_read<0>();
        if (named_bar_any(1, 256, !waited)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float o[32];
#pragma unroll 1
        for (int c = 0; c < 64; c += 32) {
          tmem_ld32(lane_base + 256 + acc * 128 + c0 + c, o);
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            uint4 pk;
            pk.x = pack_bf16x2(o[j], o[j + 1]);
            pk.y = pack_bf16x2(o[j + 2], o[j + 3]);
            pk.z = pack_bf16x2(o[j + 4], o[j + 5]);
            pk.w = pack_bf16x2(o[j + 6], o[j + 7]);
            *reinterpret_cast<uint4*>(x_tile + swz128_offset_bf16(v, c0 + c + j, kBoxBytes)) = pk;
          }
        }
        tc_fence_before();
        mbar_arrive(&o_empty[acc]);
        fence_async_smem();
        named_bar(1, 256);
        if (leader) {
          tma_store_4d(&tm_o, x_tile, 0, h, tile * kRowsPerTile, b, pol_out);
          tma_store_4d(&tm_o, x_tile + kBoxBytes, 64, h, tile * kRowsPerTile, b, pol_out);
          bulk_commit();
        }
      }
    }
    if (leader) bulk_wait_all();
    if (!ok) {
      record_error(kErrTimeout);
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

}  // namespace gdn
