// State chain: S_t = gamma_t * (S_{t-1} - beta_t * S_{t-1} A_t) + beta_t * B_t, frame after
// frame, one CTA per (batch, head). This is the only serial dependency of the layer, so the
// kernel is built for per-frame latency:
//
//   * The identity part of the frame map is kept implicit and exact: S lives in fp32 registers
//     of 16 epilogue warps (thread = one row v of S, a quarter of its columns); only the small
//     correction S_{t-1} A_t goes through the tensor core (S as a bf16 K-major operand written
//     by the epilogue into shared memory, A_t as a bf16 K-major operand loaded by TMA through a
//     4-stage ring, f32 accumulate in TMEM).
//   * B_t never touches shared memory: it is stored in the four-key interleaved layout of
//     b4_index, so each epilogue warp loads its 32 rows x 4 keys as 512 contiguous bytes, and
//     each thread loads its slice one frame ahead, into registers.
//   * A storer warp TMA-stores each S_t (the bf16 operand tile, which is exactly the bf16 copy
//     of the state the output GEMM needs) and does all hand-off bookkeeping, so the MMA warp
//     only waits for the tile and A_t and issues the MMAs.
//
// Warps: 0..15 epilogue (warp w: rows 32*(w%4).., columns (w/4)*DP/4..), 16 TMA producer,
// 17 TMEM allocator + MMA issuer, 18 storer.
//
// Standalone (gdn_chain_kernel): A_t, B_t, S_t at workspace row (b*H+h)*T + t; A_t, B_t of
// later frames are prefetched into L2. Fused (chain role of gdn_fused_kernel, CTA
// base + b*H + h): rows (b*H+h)*R + t%R of the rings; frame t is read once stats_flag says it
// is there, S_t is stored into its slot once the output of frame t-R has released it, and
// chain_prog is advanced after each store has completed.
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace gdn {

template <int DP>
struct ChainLayout {
  static constexpr int kABytes = DP * DP * 2;   // A_t bf16: DP/64 blocks of DP rows x 128 B
  static constexpr int kStages = 4;
  static constexpr int kSBlockBytes = 128 * 128;          // S operand: 128 rows x 64 cols bf16
  static constexpr int kSBytes = (DP / 64) * kSBlockBytes;
  static constexpr int kEpiWarps = 16;
  static constexpr int kThreads = (kEpiWarps + 3) * 32;
  static constexpr int kWarpProducer = kEpiWarps;
  static constexpr int kWarpMma = kEpiWarps + 1;
  static constexpr int kWarpStorer = kEpiWarps + 2;
  static constexpr int kCols = DP / 4;  // columns of S per epilogue thread
  static constexpr int kTmemCols = 128;
  static constexpr int kSmemBytes = kStages * kABytes + kSBytes + 512 + 1024;
};

template <int DP, bool kFused>
__device__ __forceinline__ void chain_body(const CUtensorMap* tm_a, const float* __restrict__ B_ws,
                                           const CUtensorMap* tm_s,
                                           const float* __restrict__ gamma,
                                           const float* __restrict__ beta,
                                           const float* __restrict__ state_in,
                                           float* __restrict__ state_out, const Problem& p,
                                           const Handoff& hf, uint8_t* smem) {
  using L = ChainLayout<DP>;
  uint8_t* s_tile = smem + L::kStages * L::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(s_tile + L::kSBytes);
  uint64_t* empty = full + L::kStages;
  uint64_t* b_ready = empty + L::kStages;  // B_t of the stage's frame may be read
  uint64_t* mma_done = b_ready + L::kStages;
  uint64_t* s_ready = mma_done + 1;        // the S tile holds the new state
  uint64_t* s_stored = s_ready + 1;        // the TMA store of the S tile has read it
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_stored + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int bh = kFused ? static_cast<int>(blockIdx.x) - hf.base : static_cast<int>(blockIdx.x);
  const int b = bh / p.H;
  const int h = bh - b * p.H;
  const int T = p.T;
  const int D = p.D;
  // row of frame f's A_t / B_t / S_t
  auto row_of = [&](int f) { return kFused ? bh * hf.R + f % hf.R : bh * T + f; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&b_ready[s], 1);
    }
    mbar_init(mma_done, 1);
    mbar_init(s_ready, L::kEpiWarps * 32);
    mbar_init(s_stored, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == L::kWarpMma) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == L::kWarpProducer) {
    // ---------------------------------------------------------------- A_t via TMA, B_t gate
    if (elect_one()) {
      tma_prefetch_desc(tm_a);
      const uint64_t pol = kFused ? policy_evict_last() : policy_evict_first();
      constexpr int kPrefetch = 8;  // standalone: frames pulled into L2 ahead of use
      auto prefetch = [&](int f) {
#pragma unroll
        for (int kb = 0; kb < DP / 64; ++kb) tma_prefetch_3d(tm_a, kb * 64, 0, row_of(f));
        bulk_prefetch_l2(B_ws + static_cast<long>(row_of(f)) * D * D,
                         static_cast<uint32_t>(D * D * 4));
      };
      if constexpr (!kFused)
        for (int f = 0; f < kPrefetch && f < T; ++f) prefetch(f);
      for (int t = 0; t < T; ++t) {
        const int stage = t % L::kStages;
        const uint32_t phase = (t / L::kStages) & 1;
        if constexpr (!kFused) {
          if (t + kPrefetch < T) prefetch(t + kPrefetch);
        }
        if (!mbar_wait(&empty[stage], phase ^ 1)) {
          give_up(hf, abort_flag);
          break;
        }
        if constexpr (kFused) {
          if (!wait_flag_ge(hf.stats_flag + static_cast<long>(bh) * T + t, 1, hf.abort)) {
            give_up(hf, abort_flag);
            break;
          }
          fence_async_global();
        }
        mbar_arrive(&b_ready[stage]);
        mbar_arrive_expect_tx(&full[stage], L::kABytes);
        uint8_t* st = smem + stage * L::kABytes;
        const int row = row_of(t);
#pragma unroll
        for (int kb = 0; kb < DP / 64; ++kb)
          tma_load_3d(st + kb * DP * 128, tm_a, &full[stage], kb * 64, 0, row, pol);
      }
    }
  } else if (warp == L::kWarpMma) {
    // ---------------------------------------------------------------- MMA: P = S_{t-1} A_t
    constexpr uint32_t idesc = idesc_bf16(128, DP, false, false);
    const uint32_t s_base = smem_u32(s_tile);
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int stage = t % L::kStages;
      const uint32_t phase = (t / L::kStages) & 1;
      if (!mbar_wait(&full[stage], phase) || !mbar_wait(s_ready, t & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (elect_one()) {
        const uint32_t a_base = smem_u32(smem + stage * L::kABytes);
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
        mma_commit(&empty[stage]);
      }
      __syncwarp();
    }
    if (!ok) give_up(hf, abort_flag);
  } else if (warp == L::kWarpStorer) {
    // ---------------------------------------------------------------- S_t -> global, hand-off
    if (elect_one()) {
      tma_prefetch_desc(tm_s);
      const uint64_t pol_s = policy_evict_last();
      // Phase 0 of s_ready is the initial state. Wait for it first: a parity wait only tells the
      // current phase from the previous one, so every phase must be waited for in order.
      bool ok = mbar_wait(s_ready, 0);
      for (int f = 0; f < T && ok; ++f) {
        // the tile holds S_f once the epilogue's (f+1)-th arrival completes s_ready
        if (!mbar_wait(s_ready, (f + 1) & 1)) {
          ok = false;
          break;
        }
        if constexpr (kFused) {
          // the slot of frame f last held S_{f-R}; its output must have loaded it
          if (f >= hf.R &&
              !wait_flag_ge(hf.out_flag + static_cast<long>(bh) * T + f - hf.R, 1, hf.abort)) {
            ok = false;
            mbar_arrive(s_stored);
            break;
          }
        }
#pragma unroll
        for (int kb = 0; kb < DP / 64; ++kb)
          tma_store_3d(tm_s, s_tile + kb * L::kSBlockBytes, kb * 64, 0, row_of(f), pol_s);
        bulk_commit();
        bulk_wait_read<0>();
        mbar_arrive(s_stored);
        if constexpr (kFused) {
          bulk_wait_all();
          fence_async_global();
          st_release(hf.chain_prog + bh, f + 1);
        }
      }
      bulk_wait_all();
      if (!ok) give_up(hf, abort_flag);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (512 threads)
    const uint32_t quarter = warp & 3;
    const int v = quarter * 32 + lane;              // row of S (value index)
    const int c0 = (warp >> 2) * L::kCols;          // first column (key index) owned
    const uint32_t taddr = tmem_base + ((quarter * 32) << 16) + c0;
    const bool row_ok = v < D;
    float S[L::kCols];
    float Bv[L::kCols];
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
    // B_f slice of this thread, from L2 (never L1: ring slots are rewritten)
    auto load_b = [&](int f) {
      const float* bm = B_ws + static_cast<long>(row_of(f)) * D * D;
#pragma unroll
      for (int j = 0; j < L::kCols; j += 4) {
        const int col = c0 + j;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (row_ok && col < D) x = __ldcg(reinterpret_cast<const float4*>(bm + b4_index(v, col, D)));
        Bv[j] = x.x;
        Bv[j + 1] = x.y;
        Bv[j + 2] = x.z;
        Bv[j + 3] = x.w;
      }
    };
    write_s_tile();
    fence_async_smem();
    tc_fence_before();
    bool ok = mbar_wait(&b_ready[0], 0);
    mbar_arrive(s_ready);
    if (ok) load_b(0);

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
    for (int t = 0; t < T && ok; ++t) {
      if ((t & 31) == 0) {
        g_cur = g_next;
        b_cur = b_next;
        load_gb((t >> 5) + 1, g_next, b_next);
      }
      const float g = __shfl_sync(0xffffffffu, g_cur, t & 31);
      const float be = __shfl_sync(0xffffffffu, b_cur, t & 31);
      if (!mbar_wait(mma_done, t & 1) || (t > 0 && !mbar_wait(s_stored, (t - 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float gbe = g * be;
#pragma unroll
      for (int c = 0; c < L::kCols; c += 16) {
        float P[16];
        tmem_ld16(taddr + c, P);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          S[c + j] = fmaf(g, S[c + j], fmaf(be, Bv[c + j], -gbe * P[j]));
      }
      write_s_tile();
      fence_async_smem();
      tc_fence_before();
      // wait for frame t+1's gate before completing s_ready: the producer can only re-arm this
      // stage's b_ready after the MMA of frame t+1, which needs this s_ready
      if (t + 1 < T && !mbar_wait(&b_ready[(t + 1) % L::kStages], ((t + 1) / L::kStages) & 1)) {
        ok = false;
        mbar_arrive(s_ready);
        break;
      }
      mbar_arrive(s_ready);
      if (t + 1 < T) load_b(t + 1);
    }
    if (!ok) give_up(hf, abort_flag);
    if (state_out != nullptr && row_ok) {
      float* so = state_out + (static_cast<long>(bh) * D + v) * D;
#pragma unroll
      for (int j = 0; j < L::kCols; j += 4)
        if (c0 + j < D)
          *reinterpret_cast<float4*>(so + c0 + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == L::kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

template <int DP>
__global__ void __launch_bounds__(ChainLayout<DP>::kThreads, 1)
    gdn_chain_kernel(const __grid_constant__ CUtensorMap tm_a, const float* __restrict__ B_ws,
                     const __grid_constant__ CUtensorMap tm_s, const float* __restrict__ gamma,
                     const float* __restrict__ beta, const float* __restrict__ state_in,
                     float* __restrict__ state_out, Problem p) {
  extern __shared__ uint8_t smem_raw[];
  const Handoff none{nullptr, nullptr, nullptr, nullptr, 1, 0, 0};
  chain_body<DP, false>(&tm_a, B_ws, &tm_s, gamma, beta, state_in, state_out, p, none,
                        align1k(smem_raw));
}

}  // namespace gdn
