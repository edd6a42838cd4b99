// State chain: S_t = gamma_t * (S_{t-1} - beta_t * S_{t-1} A_t) + beta_t * B_t, frame after
// frame, one CTA per (batch, head).
//
// The identity part of the frame map is kept implicit and exact: S lives in fp32 registers of
// the epilogue threads (thread = one row v of S, half of its columns), and only the small
// correction S_{t-1} A_t goes through the tensor core (S as a bf16 K-major operand written by
// the epilogue into shared memory, A_t as a bf16 K-major operand loaded by TMA, f32
// accumulate in TMEM). B_t (f32) arrives by TMA in 128B-swizzled 32-column blocks so that each
// thread reads its own row without bank conflicts. Each S_t is written to the workspace as a
// bf16 row-major D x D matrix (the operand of the output GEMM) by one TMA store of the bf16
// operand tile, issued by the MMA thread before it reads the same tile for the next frame.
//
// Warp roles: warp 0 TMA producer (A_t, B_t, two stages, one frame ahead), warp 1 TMEM
// allocator + MMA issuer, warps 2..9 epilogue (warp w owns rows 32*(w%4).. and column half
// (w-2)/4).
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace gdn {

template <int DP>
struct ChainLayout {
  static constexpr int kABytes = DP * DP * 2;   // A_t bf16: DP/64 blocks of DP rows x 128 B
  static constexpr int kBBytes = DP * DP * 4;   // B_t f32 : DP/32 blocks of DP rows x 128 B
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = 2;
  static constexpr int kSBlockBytes = 128 * 128;          // S operand: 128 rows x 64 cols bf16
  static constexpr int kSBytes = (DP / 64) * kSBlockBytes;
  static constexpr int kThreads = 320;
  static constexpr int kCols = DP / 2;  // columns of S per epilogue thread
  static constexpr int kTmemCols = 128;
  static constexpr int kSmemBytes = kStages * kStageBytes + kSBytes + 512 + 1024;
};

template <int DP>
__global__ void __launch_bounds__(ChainLayout<DP>::kThreads, 1)
    gdn_chain_kernel(const __grid_constant__ CUtensorMap tm_a,
                     const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_s, const float* __restrict__ gamma,
                     const float* __restrict__ beta, const float* __restrict__ state_in,
                     float* __restrict__ state_out, Problem p) {
  using L = ChainLayout<DP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1k(smem_raw);
  uint8_t* s_tile = smem + L::kStages * L::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(s_tile + L::kSBytes);
  uint64_t* empty = full + L::kStages;
  uint64_t* mma_done = empty + L::kStages;
  uint64_t* s_ready = mma_done + 1;
  uint64_t* s_stored = s_ready + 1;  // the TMA store of the S tile has read it
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_stored + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int bh = blockIdx.x;
  const int b = bh / p.H;
  const int h = bh - b * p.H;
  const int T = p.T;
  const int D = p.D;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 256);
    }
    mbar_init(mma_done, 1);
    mbar_init(s_ready, 256);
    mbar_init(s_stored, 1);
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
    if (elect_one()) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      const uint64_t pol = policy_evict_first();
      // pull A_t and B_t of frames kPrefetch ahead into L2 so the per-frame loads below hit L2
      constexpr int kPrefetch = 8;
      auto prefetch = [&](int f) {
#pragma unroll
        for (int kb = 0; kb < DP / 64; ++kb) tma_prefetch_3d(&tm_a, kb * 64, 0, bh * T + f);
#pragma unroll
        for (int cb = 0; cb < DP / 32; ++cb) tma_prefetch_3d(&tm_b, cb * 32, 0, bh * T + f);
      };
      for (int f = 0; f < kPrefetch && f < T; ++f) prefetch(f);
      int stage = 0;
      uint32_t phase = 0;
      for (int t = 0; t < T; ++t) {
        if (t + kPrefetch < T) prefetch(t + kPrefetch);
        if (!mbar_wait(&empty[stage], phase ^ 1)) {
          record_error(kErrTimeout);
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&full[stage], L::kStageBytes);
        uint8_t* st = smem + stage * L::kStageBytes;
        const int row = bh * T + t;
#pragma unroll
        for (int kb = 0; kb < DP / 64; ++kb)
          tma_load_3d(st + kb * DP * 128, &tm_a, &full[stage], kb * 64, 0, row, pol);
#pragma unroll
        for (int cb = 0; cb < DP / 32; ++cb)
          tma_load_3d(st + L::kABytes + cb * DP * 128, &tm_b, &full[stage], cb * 32, 0, row,
                      pol);
        if (++stage == L::kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  } else if (warp == 1) {
    constexpr uint32_t idesc = idesc_bf16(128, DP, false, false);
    const uint32_t s_base = smem_u32(s_tile);
    const uint64_t pol_s = policy_evict_last();
    if (lane == 0) tma_prefetch_desc(&tm_s);
    // The S tile holds S_{t-1} when step t starts; store it as frame t-1's state (t >= 1),
    // then multiply it by A_t. The epilogue overwrites the tile only after both the MMAs
    // (mma_done) and the store's read of the tile (s_stored) are complete.
    auto store_tile = [&](int frame) {
#pragma unroll
      for (int kb = 0; kb < DP / 64; ++kb)
        tma_store_3d(&tm_s, s_tile + kb * L::kSBlockBytes, kb * 64, 0, bh * T + frame, pol_s);
      bulk_commit();
    };
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      if (!mbar_wait(&full[stage], phase) || !mbar_wait(s_ready, t & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (elect_one()) {
        if (t > 0) store_tile(t - 1);
        const uint32_t a_base = smem_u32(smem + stage * L::kStageBytes);
#pragma unroll
        for (int kb = 0; kb < DP / 64; ++kb) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t da = smem_desc(s_base + kb * L::kSBlockBytes + ks * 32, 16, 1024);
            const uint64_t db = smem_desc(a_base + kb * DP * 128 + ks * 32, 16, 1024);
            mma_bf16(tmem_base, da, db, idesc, (kb | ks) != 0);
          }
        }
        mma_commit(mma_done);
        bulk_wait_read<0>();
        mbar_arrive(s_stored);
      }
      __syncwarp();
      if (++stage == L::kStages) {
        stage = 0;
        phase ^= 1;
      }
    }
    // the last state S_{T-1}
    if (ok && !mbar_wait(s_ready, T & 1)) ok = false;
    if (elect_one()) {
      if (ok) store_tile(T - 1);
      bulk_wait_all();
    }
    __syncwarp();
    if (!ok) {
      record_error(kErrTimeout);
      *abort_flag = 1;
    }
  } else {
    // ---------------------------------------------------------------- epilogue (256 threads)
    const uint32_t quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int v = quarter * 32 + lane;  // row of S (value index)
    const int c0 = half * L::kCols;     // first column (key index) owned
    const uint32_t taddr = tmem_base + ((quarter * 32) << 16) + c0;
    const bool row_ok = v < D;
    float S[L::kCols];
    const float* sin = state_in ? state_in + (static_cast<long>(bh) * D + v) * D : nullptr;
#pragma unroll
    for (int j = 0; j < L::kCols; ++j) {
      const int col = c0 + j;
      S[j] = (sin != nullptr && row_ok && col < D) ? sin[col] : 0.f;
    }
    auto write_s_tile = [&]() {
#pragma unroll
      for (int j = 0; j < L::kCols; j += 8) {
        uint4 pk;
        pk.x = pack_bf16x2(S[j], S[j + 1]);
        pk.y = pack_bf16x2(S[j + 2], S[j + 3]);
        pk.z = pack_bf16x2(S[j + 4], S[j + 5]);
        pk.w = pack_bf16x2(S[j + 6], S[j + 7]);
        *reinterpret_cast<uint4*>(s_tile + swz128_offset_bf16(v, c0 + j, L::kSBlockBytes)) = pk;
      }
    };
    write_s_tile();
    fence_async_smem();
    tc_fence_before();
    mbar_arrive(s_ready);

    int stage = 0;
    uint32_t phase = 0;
    // gamma_t, beta_t: each lane holds frame (32*blk + lane) of the current and next block of
    // 32 frames; the value for frame t is shuffled from lane t % 32.
    const long gb_base = static_cast<long>(b) * T * p.H + h;
    auto load_gb = [&](int blk, float& gv, float& bv) {
      const int f = blk * 32 + static_cast<int>(lane);
      gv = f < T ? __ldg(gamma + gb_base + static_cast<long>(f) * p.H) : 0.f;
      bv = f < T ? __ldg(beta + gb_base + static_cast<long>(f) * p.H) : 0.f;
    };
    float g_cur, b_cur, g_next, b_next;
    load_gb(0, g_next, b_next);
    for (int t = 0; t < T; ++t) {
      if ((t & 31) == 0) {
        g_cur = g_next;
        b_cur = b_next;
        load_gb((t >> 5) + 1, g_next, b_next);
      }
      const float g = __shfl_sync(0xffffffffu, g_cur, t & 31);
      const float be = __shfl_sync(0xffffffffu, b_cur, t & 31);
      if (!mbar_wait(mma_done, t & 1) || !mbar_wait(&full[stage], phase) ||
          !mbar_wait(s_stored, t & 1)) {
        record_error(kErrTimeout);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      float P[L::kCols];
#pragma unroll
      for (int c = 0; c < L::kCols / 32; ++c) tmem_ld32(taddr + c * 32, P + c * 32);
      const uint8_t* bt = smem + stage * L::kStageBytes + L::kABytes;
#pragma unroll
      for (int j = 0; j < L::kCols; j += 4) {
        // rows v >= DP are M-padding of the MMA (DP == 64): no B_t row, S stays 0 there
        const float4 bv =
            (v < DP) ? *reinterpret_cast<const float4*>(bt + swz128_offset_f32(v, c0 + j, DP * 128))
                     : make_float4(0.f, 0.f, 0.f, 0.f);
        S[j] = g * (S[j] - be * P[j]) + be * bv.x;
        S[j + 1] = g * (S[j + 1] - be * P[j + 1]) + be * bv.y;
        S[j + 2] = g * (S[j + 2] - be * P[j + 2]) + be * bv.z;
        S[j + 3] = g * (S[j + 3] - be * P[j + 3]) + be * bv.w;
      }
      write_s_tile();
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(s_ready);
      mbar_arrive(&empty[stage]);
      if (++stage == L::kStages) {
        stage = 0;
        phase ^= 1;
      }
    }
    if (state_out != nullptr && row_ok) {
      float* so = state_out + (static_cast<long>(bh) * D + v) * D;
#pragma unroll
      for (int j = 0; j < L::kCols; j += 4)
        if (c0 + j < D) *reinterpret_cast<float4*>(so + c0 + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
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
