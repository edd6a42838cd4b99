// Single-frame streaming step, for every (batch, head) of one launch:
//
//   A = s^2 K^T K,  B = s V^T K        (tcgen05, K and V tiles MN-major from TMA)
//   P = S_in A                          (tcgen05, S_in and A as bf16 core-matrix tiles)
//   S_out = gamma (S_in - beta P) + beta B   (fp32, identity part exact)
//   O = Q S_out^T                       (tcgen05, S_out as the bf16 B operand)
//
// Work is split into units taken dynamically from one counter, so that the 2.2 (batch, head)
// items per SM of the 16-stream x 20-head workload do not leave most of the GPU idle during a
// last partial wave:
//   * statistics units (one per item, numbered first): A, B, the update, state_out, and the
//     item's updated state S' as a bf16 operand tile, bulk-copied to global memory and published
//     with a release flag;
//   * output units (up to kOutTiles token tiles of one item, numbered after all statistics
//     units): wait for the item's flag, bulk-load S', and compute O for their tiles.
// Every output unit's statistics unit has a smaller number, so some CTA took it earlier and it
// never waits on anything an output unit does; with all CTAs co-resident (cooperative launch)
// the flag waits cannot deadlock, and every wait is bounded.
//
// Shared memory: a ring of 32 KB stages (K, V and Q tiles, 128 tokens x 128 dims bf16), the S
// tile (S_in, then S' for the copy out, as 8-row x 16 B core matrices), the X tile (A as core
// matrices; the bf16 output staging of the TMA stores), the O tile (S' of the current output
// unit). TMEM: columns [0,128) A then P, [128,256) B, [256,512) two output accumulators.
//
// Warps: 0 TMA producer and work distribution, 1 TMEM allocator + MMA issuer, 2..9 epilogue
// (warp w: rows 32*(w%4).., column half (w-2)/4).
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace gdn {

struct StepLayout {
  static constexpr int kStageBytes = 2 * kBoxBytes;  // 128 x 128 bf16 tile (two TMA boxes)
  static constexpr int kStages = 4;
  static constexpr int kTileBytes = 128 * 128 * 2;   // S, X and O tiles
  static constexpr int kOutTiles = 4;                // token tiles per output unit
  static constexpr int kThreads = 320;
  static constexpr int kTmemCols = 512;
  static constexpr int kSmemBytes = kStages * kStageBytes + 3 * kTileBytes + 512 + 1024;
};

// Hand-off between the units of one launch. The flag words persist across launches: `ready`
// holds the number of the launch that last published the item (epochs, so nothing is cleared
// between launches), and the last CTA to finish resets the counters for the next launch.
struct StepShared {
  int* ready;       // [B*H] = epoch once the item's S' tile of this launch is in sprime
  int* next_unit;   // work counter (0 at launch)
  int* done;        // CTAs finished (0 at launch)
  int* abort;       // set by the first CTA that gives up a wait (0 at launch)
  uint8_t* sprime;  // [B*H] S' tiles (kTileBytes each, core-matrix layout of s8_offset_bytes)
  int epoch;        // this launch's number, >= 1 and increasing
};

// q, k, v, out tensor maps over [B, 1, N, H, D] (T = 1); gamma, beta [B, H]; state [B, H, D, D].
__global__ void __launch_bounds__(StepLayout::kThreads, 1)
    gdn_step_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_o, const float* __restrict__ gamma,
                    const float* __restrict__ beta, const float* state_in, float* state_out,
                    Problem p, StepShared sh) {
  using L = StepLayout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1k(smem_raw);
  uint8_t* s_tile = smem + L::kStages * L::kStageBytes;
  uint8_t* x_tile = s_tile + L::kTileBytes;
  uint8_t* o_tile = x_tile + L::kTileBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(o_tile + L::kTileBytes);
  uint64_t* empty = full + L::kStages;
  uint64_t* stats_done = empty + L::kStages;  // A, B accumulated
  uint64_t* sa_ready = stats_done + 1;        // S tile and A tile written
  uint64_t* p_done = sa_ready + 1;            // P = S A accumulated
  uint64_t* s2_ready = p_done + 1;            // P and B read out of TMEM
  uint64_t* os_full = s2_ready + 1;           // S' of the current output unit loaded
  uint64_t* os_free = os_full + 1;            // the output unit's MMAs are done with the O tile
  uint64_t* o_full = os_free + 1;             // [2]
  uint64_t* o_empty = o_full + 2;             // [2]
  uint64_t* mma_drain = o_empty + 2;
  ItemRing ring{reinterpret_cast<int*>(mma_drain + 1 + 8), mma_drain + 1};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ring.ids + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const long n_items = static_cast<long>(p.B) * p.H;
  const int n_tiles = (p.N + kRowsPerTile - 1) / kRowsPerTile;
  const int n_opi = (n_tiles + L::kOutTiles - 1) / L::kOutTiles;  // output units per item
  const long n_units = n_items * (1 + n_opi);
  const int D = p.D;
  const Handoff hf{nullptr, nullptr, nullptr, sh.abort, sh.next_unit, 1, 1, -1, 0, 0};
  // unit u: statistics of item u (u < n_items), else tiles [t0, t1) of an item's output
  struct Unit {
    bool stats;
    long item;
    int t0, t1;
  };
  auto decode = [&](long u) {
    Unit x;
    x.stats = u < n_items;
    if (x.stats) {
      x.item = u;
      x.t0 = 0;
      x.t1 = n_tiles;
    } else {
      const long o = u - n_items;
      x.item = o / n_opi;
      x.t0 = static_cast<int>(o - x.item * n_opi) * L::kOutTiles;
      x.t1 = min(n_tiles, x.t0 + L::kOutTiles);
    }
    return x;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(stats_done, 1);
    mbar_init(sa_ready, 256);
    mbar_init(p_done, 1);
    mbar_init(s2_ready, 256);
    mbar_init(os_full, 1);
    mbar_init(os_free, 1);
    for (int a = 0; a < 2; ++a) {
      mbar_init(&o_full[a], 1);
      mbar_init(&o_empty[a], 256);
    }
    mbar_init(mma_drain, 1);
    for (int i = 0; i < 8; ++i) mbar_init(&ring.bars[i], 1);
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
    // ---------------------------------------------------------------- work + TMA producer
    if (elect_one()) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const uint64_t pol = policy_evict_first();
      const uint64_t pol_s = policy_evict_last();
      StageFills<L::kStages> fills;
      StageFills<1> os_fills;
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
      int lo = 0;  // output units taken by this CTA
      for (int li = 0; ok && !*abort_flag; ++li) {
        const long u = ring.produce(li, sh.next_unit, n_units);
        if (u < 0) break;
        const Unit x = decode(u);
        const int h = static_cast<int>(x.item % p.H);
        const int b = static_cast<int>(x.item / p.H);
        if (x.stats) {
          for (int tile = 0; tile < n_tiles && ok; ++tile)
            ok = load_tile(&tm_k, h, tile, b) && load_tile(&tm_v, h, tile, b);
        } else {
          // the item's S', published by the CTA that ran its statistics unit
          ok = wait_flag_ge(sh.ready + x.item, sh.epoch, sh.abort);
          fence_async_global();
          ok = ok && (lo == 0 || mbar_wait(os_free, (lo - 1) & 1));
          if (ok) {
            mbar_arrive_expect_tx(os_full, L::kTileBytes);
            bulk_load(o_tile, sh.sprime + x.item * L::kTileBytes, L::kTileBytes, os_full, pol_s);
            os_fills.filled(0, lo & 1);
          }
          for (int tile = x.t0; tile < x.t1 && ok; ++tile) ok = load_tile(&tm_q, h, tile, b);
          ++lo;
        }
      }
      if (!ok) give_up(hf, abort_flag);
      fills.drain(full);
      os_fills.drain(os_full);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc_stats = idesc_bf16(128, 128, true, true);
    constexpr uint32_t idesc_kmaj = idesc_bf16(128, 128, false, false);
    const uint32_t s_base = smem_u32(s_tile);
    const uint32_t x_base = smem_u32(x_tile);
    const uint32_t o_base = smem_u32(o_tile);
    const uint32_t t_a = tmem_base, t_b = tmem_base + 128, t_o = tmem_base + 256;
    int stage = 0;
    uint32_t phase = 0;
    int tc = 0, ls = 0, lo = 0;
    bool ok = true;
    auto next_stage = [&]() {
      if (++stage == L::kStages) {
        stage = 0;
        phase ^= 1;
      }
    };
    for (int li = 0; ok; ++li) {
      const long u = ring.consume(li);
      if (u == -2) ok = false;
      if (u < 0) break;
      const Unit x = decode(u);
      if (x.stats) {
        // the previous statistics unit's epilogue has read P and B: A, B may be rewritten
        if (ls > 0 && !mbar_wait(s2_ready, (ls - 1) & 1)) {
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
        if (!mbar_wait(sa_ready, ls & 1)) {
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
        ++ls;
      } else {
        // O = Q S'^T for the unit's tiles
        if (!mbar_wait(os_full, lo & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int tile = x.t0; tile < x.t1; ++tile, ++tc) {
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
              const uint64_t db = smem_desc_noswz(o_base + ks * 2 * 2048, 2048, 128);
              mma_bf16(t_o + acc * 128, da, db, idesc_kmaj, ks != 0);
            }
            mma_commit(&empty[stage]);
            mma_commit(&o_full[acc]);
          }
          __syncwarp();
          next_stage();
        }
        if (!ok) break;
        if (elect_one()) mma_commit(os_free);
        __syncwarp();
        ++lo;
      }
    }
    if (!ok) give_up(hf, abort_flag);
    if (elect_one()) mma_commit(mma_drain);
    __syncwarp();
    mbar_wait(mma_drain, 0);
  } else {
    // ---------------------------------------------------------------- epilogue (256 threads)
    const uint32_t quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int v = quarter * 32 + lane;  // row: value index of S, key index k' of A
    const int c0 = half * 64;           // first column owned
    const uint32_t lane_base = tmem_base + ((quarter * 32) << 16);
    const bool row_ok = v < D;
    const bool leader = (threadIdx.x == 64);
    const float s = p.key_scale;
    const float s2 = s * s;
    const uint64_t pol_out = policy_evict_first();
    if (leader) tma_prefetch_desc(&tm_o);
    auto core_off = [&](int col) { return (col >> 3) * 2048 + v * 16; };  // 8-column group
    int tc = 0, ls = 0;
    bool ok = true;
    for (int li = 0; ok; ++li) {
      const long u = ring.consume(li);
      if (named_bar_any(1, 256, u == -2)) {
        ok = false;
        break;
      }
      if (u < 0) break;
      const Unit x = decode(u);
      const long bh = x.item;
      const int h = static_cast<int>(bh % p.H);
      const int b = static_cast<int>(bh / p.H);
      if (x.stats) {
        const float g = __ldg(gamma + bh);
        const float be = __ldg(beta + bh);
        // S_in row v, this thread's 64 columns (fp32, kept for the update)
        float S[64];
        const float* sin = state_in ? state_in + (bh * D + v) * D : nullptr;
#pragma unroll
        for (int j = 0; j < 64; j += 4) {
          const int col = c0 + j;
          float4 xv = make_float4(0.f, 0.f, 0.f, 0.f);
          if (sin != nullptr && row_ok && col < D) xv = *reinterpret_cast<const float4*>(sin + col);
          S[j] = xv.x;
          S[j + 1] = xv.y;
          S[j + 2] = xv.z;
          S[j + 3] = xv.w;
        }
        // the X tile is free once an earlier output unit's last store has read it; the S tile
        // once the previous statistics unit's copy-out has completed (the leader waited for it
        // before reaching this barrier)
        const bool bad = !mbar_wait(stats_done, ls & 1);
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
        if (named_bar_any(1, 256, !mbar_wait(p_done, ls & 1))) {
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
        tc_fence_before();
        mbar_arrive(s2_ready);
        if (state_out != nullptr && row_ok) {
          float* so = state_out + (bh * D + v) * D;
#pragma unroll
          for (int j = 0; j < 64; j += 4)
            if (c0 + j < D)
              *reinterpret_cast<float4*>(so + c0 + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
        }
        // S' as the bf16 operand tile of the output units, copied out and published
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
        named_bar(1, 256);
        if (leader) {
          bulk_store(sh.sprime + bh * L::kTileBytes, s_tile, L::kTileBytes);
          bulk_commit();
          bulk_wait_all();
          // the copy's writes (async proxy) before the flag (generic release at GPU scope)
          fence_async_global();
          st_release(sh.ready + bh, sh.epoch);
        }
        ++ls;
      } else {
        // output tiles through the X tile as TMA-store staging (128B-swizzled, two boxes)
        for (int tile = x.t0; tile < x.t1; ++tile, ++tc) {
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
    }
    if (leader) bulk_wait_all();
    if (!ok) give_up(hf, abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
  // the last CTA out resets the launch's counters (no CTA takes work or reads abort any more)
  if (threadIdx.x == 0 && atomicAdd(sh.done, 1) == static_cast<int>(gridDim.x) - 1) {
    *sh.next_unit = 0;
    *sh.abort = 0;
    *sh.done = 0;
  }
}

}  // namespace gdn
