// Frame statistics: for every frame t of every head, in parallel,
//   GDN: A_t = s^2 K_t^T K_t  (stored bf16, D x D, row k', column k)
//        B_t = s   V_t^T K_t  (stored f32,  D x D, row v,  column k)
//   LA : B_t = [V_t | 1]^T relu(K_t)  (stored f32, (D+1) x D; row D is sum relu(k), the
//        normaliser contribution)
// as tcgen05 GEMMs contracting over the N tokens of the frame. K and V tiles (128 tokens x 64
// dims per TMA box, 128B-swizzled) are both MMA operands in MN-major form, so the transposes
// cost nothing. Accumulators live in TMEM (double-buffered across work items so the epilogue
// of one frame overlaps the MMAs of the next).
//
// Warp roles (one CTA per SM, persistent over work items):
//   warp 0      TMA producer (one elected thread)
//   warp 1      TMEM allocator + MMA issuer (one elected thread)
//   warps 2..5  epilogue: TMEM -> registers -> scale -> global (LA: per-block sums)
//   warps 6..   (LA, fp8 and RoPE only) in-place transform of each K/V stage: relu(K) and a
//               ones column in V (LA, warps 6..9), or e4m3 -> bf16 conversion of K and V (fp8
//               inputs, DP = 128, warps 6..13, one token row of K or V per thread: the fp8
//               tiles are TMA-loaded into the second box of each bf16 operand tile), or the 3D
//               rotary embedding of the K tile (RoPE, warps 6..6+4*DP/64-1, one 64-dim box of
//               one token row per thread; V is not rotated)
//
// Standalone (gdn_stats_kernel): work item i = (b*T + t)*H + h, results at workspace row
// (b*H + h)*T + t; for LA an item is a block of frames_per_item frames (its statistics summed
// over its token rows, read through 3-D maps of the flattened (b, t, n) rows so that tiles span
// frames), results at row (b*H + h)*n_blocks + block. Fused (stats role of gdn_fused_kernel): work item i = t*B*H + (b*H + h)
// (frame-major, so the chain finds early frames first), results at ring row (b*H+h)*R + t%R,
// written only after the chain has released that slot, then published with stats_flag.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "rope_kernel.cuh"

namespace gdn {

// kRopeGroups: groups of 128 threads (4 warps) in the RoPE transform of the K tiles.
template <int DP, bool kLA, bool kF8 = false, bool kRope = false, int kRopeGroups = DP / 64>
struct StatsLayout {
  static_assert(!kF8 || (DP == 128 && !kLA), "fp8 inputs: DP = 128, GDN only");
  static_assert(!kRope || (!kF8 && !kLA), "RoPE prologue: bf16 GDN only");
  // fp8: the tensor core reads the e4m3 tiles as they land (kind::f8f6f4), no transform
  static constexpr bool kTransform = kLA || kRope;
  static constexpr int kBoxes = DP / 64;  // 64-dim boxes per bf16 operand tile
  // 128 tokens x DP dims: bf16 in kBoxes boxes, e4m3 in one 128-byte-wide box
  static constexpr int kOpBytes = kF8 ? kBoxBytes : kBoxes * kBoxBytes;
  static constexpr int kStageBytes = 2 * kOpBytes;  // K tile + V tile
  static constexpr int kStages = (DP == 128 && !kF8) ? 3 : 6;
  static constexpr int kAccCols = kLA ? 128 : (DP == 128 ? 256 : 64);
  static constexpr int kTmemCols = 2 * kAccCols;
  // LA: one K row per thread; RoPE: kRopeGroups groups of 128 threads
  static constexpr int kTransformThreads = kRope ? 128 * kRopeGroups : 128;
  static constexpr int kThreads = 192 + (kTransform ? kTransformThreads : 0);
  static constexpr int kLoadBytes = kStageBytes;  // TMA bytes per stage
  static constexpr int kBarrierBytes = 512;
  static constexpr int kTabBytes = kRope ? kRopeSmemTabBytes : 0;  // rope_stage_rc's table copy
  static constexpr int kSmemBytes = kStages * kStageBytes + kBarrierBytes + kTabBytes + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
  // barriers, item ring, TMEM slot and the fused publisher's ring within kBarrierBytes
  static_assert(8 * (3 * kStages + 4 + 8 + 1) + 32 + 8 + 8 * 16 + 32 <= kBarrierBytes, "barriers");
  static_assert(kTmemCols == 128 || kTmemCols == 256 || kTmemCols == 512, "TMEM columns");
};

struct StatsItem {
  int h, bt, bh, t;
  int nf;    // frames accumulated into this item (block-causal LA: a block of frames)
  long row;  // workspace / ring row of the results
};

// fpb: frames per item (1 for GDN; the block length for block-causal LA, whose state only needs
// each block's sum). Standalone items are (b, block, h) in that order.
template <bool kFused>
__device__ __forceinline__ StatsItem stats_item(long item, const Problem& p, const Handoff& hf,
                                                int fpb) {
  StatsItem it;
  it.nf = 1;
  if constexpr (kFused) {
    const int BH = p.B * p.H;
    it.t = static_cast<int>(item / BH);
    it.bh = static_cast<int>(item - static_cast<long>(it.t) * BH);
    const int b = it.bh / p.H;
    it.h = it.bh - b * p.H;
    it.bt = b * p.T + it.t;
    it.row = static_cast<long>(it.bh) * hf.R + it.t % hf.R;
  } else {
    const int nblk = (p.T + fpb - 1) / fpb;
    it.h = static_cast<int>(item % p.H);
    const int bj = static_cast<int>(item / p.H);
    const int b = bj / nblk;
    const int j = bj - b * nblk;
    it.t = j * fpb;
    it.nf = min(fpb, p.T - it.t);
    it.bt = b * p.T + it.t;
    it.bh = b * p.H + it.h;
    it.row = static_cast<long>(it.bh) * nblk + j;
  }
  return it;
}

// kB4: B_t stored in the four-key interleaved layout of b4_index (the chain's input) instead of
// row-major (the public gdn_frame_stats layout and the block-causal path).
template <int DP, bool kLA, bool kFused, bool kB4, bool kF8 = false, bool kRope = false,
          int kRopeGroups = DP / 64>
__device__ __forceinline__ void stats_body(const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                           __nv_bfloat16* __restrict__ A_ws,
                                           float* __restrict__ B_ws, const Problem& p,
                                           const Handoff& hf, uint8_t* smem, int fpb = 1) {
  using L = StatsLayout<DP, kLA, kF8, kRope, kRopeGroups>;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kStages * L::kStageBytes);
  uint64_t* ready = full + L::kStages;   // LA / fp8: transformed stage
  uint64_t* empty = ready + L::kStages;
  uint64_t* acc_full = empty + L::kStages;
  uint64_t* acc_empty = acc_full + 2;
  ItemRing ring{reinterpret_cast<int*>(acc_empty + 2 + 9), acc_empty + 2};  // fused only
  uint64_t* mma_drain = acc_empty + 2 + 8;  // all of this CTA's MMAs are complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ring.ids + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // fused: the epilogue hands each finished item to the publisher warp through an 8-slot ring
  // (flag index in pub_ids, one arrival per epilogue warp on pub_full; the publisher frees the
  // slot on pub_empty), so the GPU-scope release of the flag is off the epilogue's path
  uint64_t* pub_full = reinterpret_cast<uint64_t*>(tmem_slot + 2);
  uint64_t* pub_empty = pub_full + 8;
  int* pub_ids = reinterpret_cast<int*>(pub_empty + 8);
  constexpr uint32_t kPubWarp = 18;  // the fused CTA's last warp (idle in the statistics role)

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const long n_items = static_cast<long>(p.B) * ((p.T + fpb - 1) / fpb) * p.H;
  const int n_tiles = (p.N + kRowsPerTile - 1) / kRowsPerTile;
  // tiles of an item of nf frames: LA items are blocks whose nf*N token rows are contiguous in
  // the flattened (b, t, n) rows of its 3-D maps, so its tiles span frames
  auto item_tiles = [&](int nf) {
    return kLA ? (nf * p.N + kRowsPerTile - 1) / kRowsPerTile : nf * n_tiles;
  };
  const long cta0 = kFused ? blockIdx.x - hf.base : blockIdx.x;
  const long ncta = kFused ? hf.count : gridDim.x;
  // item li of this CTA: standalone a static stride, fused the role's work counter. Returns -1
  // when there are no more items, -2 on a timed-out wait.
  auto producer_item = [&](int li) -> long {
    if constexpr (kFused) return ring.produce(li, hf.next_item, n_items);
    const long it = cta0 + static_cast<long>(li) * ncta;
    return it < n_items ? it : -1;
  };
  auto consumer_item = [&](int li) -> long {
    if constexpr (kFused) return ring.consume(li);
    const long it = cta0 + static_cast<long>(li) * ncta;
    return it < n_items ? it : -1;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&ready[s], L::kTransformThreads);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 128);
    }
    for (int i = 0; i < 8; ++i) mbar_init(&ring.bars[i], 1);
    for (int i = 0; i < 8; ++i) {
      mbar_init(&pub_full[i], 4);
      mbar_init(&pub_empty[i], 1);
    }
    mbar_init(mma_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  // RoPE: the table's grid-row and grid-column entries, copied past the barriers if they fit
  RopeRc rope_rc{nullptr, 0};
  if constexpr (kRope)
    rope_rc = rope_stage_rc(
        reinterpret_cast<float2*>(smem + L::kStages * L::kStageBytes + L::kBarrierBytes), p.rope,
        threadIdx.x, blockDim.x);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (elect_one()) {
      tma_prefetch_desc(tm_k);
      tma_prefetch_desc(tm_v);
      const uint64_t pol = policy_evict_first();
      StageFills<L::kStages> fills;
      int stage = 0;
      uint32_t phase = 0;
      for (int li = 0; !*abort_flag; ++li) {
        const long item = producer_item(li);
        if (item < 0) break;
        const StatsItem it = stats_item<kFused>(item, p, hf, fpb);
        for (int ft = 0; ft < item_tiles(it.nf); ++ft) {
          const int tile = ft % n_tiles;
          const int bt = it.bt + ft / n_tiles;
          if (!mbar_wait(&empty[stage], phase ^ 1)) {
            give_up(hf, abort_flag);
            break;
          }
          mbar_arrive_expect_tx(&full[stage], L::kLoadBytes);
          uint8_t* st = smem + stage * L::kStageBytes;
          if constexpr (kLA) {
            // 128 flattened token rows from the block's first row (they may cross frames; rows
            // past the block are zeroed in K by the transform warps)
            const int row = it.bt * p.N + ft * kRowsPerTile;
#pragma unroll
            for (int j = 0; j < L::kBoxes; ++j) {
              tma_load_3d(st + j * kBoxBytes, tm_k, &full[stage], j * 64, it.h, row, pol);
              tma_load_3d(st + L::kOpBytes + j * kBoxBytes, tm_v, &full[stage], j * 64, it.h,
                          row, pol);
            }
          } else if constexpr (kF8) {
            // one 128-byte-wide e4m3 box per operand
            tma_load_4d(st, tm_k, &full[stage], 0, it.h, tile * kRowsPerTile, bt, pol);
            tma_load_4d(st + L::kOpBytes, tm_v, &full[stage], 0, it.h, tile * kRowsPerTile, bt,
                        pol);
          } else {
#pragma unroll
            for (int j = 0; j < L::kBoxes; ++j) {
              tma_load_4d(st + j * kBoxBytes, tm_k, &full[stage], j * 64, it.h,
                          tile * kRowsPerTile, bt, pol);
              tma_load_4d(st + L::kOpBytes + j * kBoxBytes, tm_v, &full[stage], j * 64, it.h,
                          tile * kRowsPerTile, bt, pol);
            }
          }
          fills.filled(stage, phase);
          if (++stage == L::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      fills.drain(full);  // this thread's copies have landed, whatever the exit path
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = kF8 ? idesc_e4m3(128, 128, true, true)
                               : kLA ? idesc_bf16(128, 128, true, true)
                                     : (DP == 128 ? idesc_bf16(128, 128, true, true)
                                                  : idesc_bf16(128, 64, true, true));
    int stage = 0;
    uint32_t phase = 0;
    for (int li = 0;; ++li) {
      const long item = consumer_item(li);
      if (item == -2) {
        give_up(hf, abort_flag);
        break;
      }
      if (item < 0) break;
      const int acc = li & 1;
      const uint32_t aph = (li >> 1) & 1;
      if (!mbar_wait(&acc_empty[acc], aph ^ 1)) {
        give_up(hf, abort_flag);
        break;
      }
      tc_fence_after();
      const uint32_t d = tmem_base + acc * L::kAccCols;
      const int nf = stats_item<kFused>(item, p, hf, fpb).nf;
      bool ok = true;
      for (int tile = 0; tile < item_tiles(nf); ++tile) {
        if (!mbar_wait(L::kTransform ? &ready[stage] : &full[stage], phase)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const uint32_t base = smem_u32(smem + stage * L::kStageBytes);
          if constexpr (kF8) {
            // e4m3 K and V tiles, both MN-major (128 dims = one 128-byte swizzle atom per token
            // row): 32 token rows (4 KB) per instruction, 8-row groups 1024 B apart
#pragma unroll
            for (int ks = 0; ks < kRowsPerTile / 32; ++ks) {
              const uint32_t accum = (tile | ks) != 0;
              const uint64_t dk = smem_desc(base + ks * 32 * 128, kBoxBytes, 1024);
              const uint64_t dv = smem_desc(base + L::kOpBytes + ks * 32 * 128, kBoxBytes, 1024);
              mma_e4m3(d, dk, dk, idesc, accum);        // A_t = K^T K
              mma_e4m3(d + 128, dv, dk, idesc, accum);  // B_t = V^T K
            }
          } else {
#pragma unroll
            for (int ks = 0; ks < kRowsPerTile / 16; ++ks) {
              const uint32_t accum = (tile | ks) != 0;
              const uint32_t koff = ks * 16 * 128;  // 16 token rows of 128 B
              if constexpr (kLA) {
                const uint64_t dv = smem_desc(base + L::kOpBytes + koff, kBoxBytes, 1024);
                const uint64_t dk = smem_desc(base + koff, kBoxBytes, 1024);
                mma_bf16(d, dv, dk, idesc, accum);
              } else if constexpr (DP == 128) {
                const uint64_t dk = smem_desc(base + koff, kBoxBytes, 1024);
                const uint64_t dv = smem_desc(base + L::kOpBytes + koff, kBoxBytes, 1024);
                mma_bf16(d, dk, dk, idesc, accum);        // A_t = K^T K
                mma_bf16(d + 128, dv, dk, idesc, accum);  // B_t = V^T K
              } else {
                // [K | V] stacked along M (K box then V box, kOpBytes apart) times K:
                // TMEM rows 0..63 = K^T K, rows 64..127 = V^T K.
                const uint64_t da = smem_desc(base + koff, L::kOpBytes, 1024);
                const uint64_t db = smem_desc(base + koff, kBoxBytes, 1024);
                mma_bf16(d, da, db, idesc, accum);
              }
            }
          }
          mma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == L::kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) {
        give_up(hf, abort_flag);
        break;
      }
      if (elect_one()) mma_commit(&acc_full[acc]);
      __syncwarp();
    }
    // every MMA issued here has completed before TMEM is released
    if (elect_one()) mma_commit(mma_drain);
    __syncwarp();
    mbar_wait(mma_drain, 0);
  } else if (warp < 6) {
    // ---------------------------------------------------------------- epilogue
    const uint32_t quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem_base + ((quarter * 32) << 16);
    const bool leader = (threadIdx.x == 64);
    const float s = p.key_scale;
    const int D = p.D;
    const int brows = kLA ? D + 1 : D;
    for (int li = 0;; ++li) {
      const long item = consumer_item(li);
      bool lost = item == -2;
      if constexpr (kFused) lost = named_bar_any(1, 128, lost);  // uniform across the epilogue
      if (lost) {
        give_up(hf, abort_flag);
        break;
      }
      if (item < 0) {
        if constexpr (kFused) {
          // end of the items: the publisher stops at this slot
          const int ps = li & 7;
          if (li >= 8 && !mbar_wait(&pub_empty[ps], ((li >> 3) & 1) ^ 1)) {
            give_up(hf, abort_flag);
            break;
          }
          if (leader) pub_ids[ps] = -2;
          __syncwarp();
          if (lane == 0) mbar_arrive(&pub_full[ps]);
        }
        break;
      }
      const int acc = li & 1;
      const uint32_t aph = (li >> 1) & 1;
      const StatsItem it = stats_item<kFused>(item, p, hf, fpb);
      bool bad = !mbar_wait(&acc_full[acc], aph);
      if constexpr (kFused) {
        // ring slot t % R of this head is free once the chain has stored S_{t-R}
        if (leader && !bad && it.t >= hf.R)
          bad = !wait_flag_ge(hf.chain_prog + it.bh, it.t - hf.R + 1, hf.abort);
        bad = named_bar_any(1, 128, bad);
      }
      if (bad) {
        give_up(hf, abort_flag);
        break;
      }
      tc_fence_after();
      const long ws = it.row;
      const uint32_t tacc = lane_base + acc * L::kAccCols;
      float v[32];
      // fp8: the dequantisation scales of this frame's K and V enter A and B here
      float fa = s * s, fb = s;
      if constexpr (kF8) {
        const long gi = static_cast<long>(it.bt) * p.H + it.h;
        const float sk = __ldg(p.k_scale + gi), sv = __ldg(p.v_scale + gi);
        fa *= sk * sk;
        fb *= sk * sv;
      }
      if constexpr (kLA) {
        // row = value index v (row D = normaliser); columns = key index
        float* brow = B_ws + (ws * brows + row) * D;
#pragma unroll 1
        for (int c = 0; c < DP / 32; ++c) {
          tmem_ld32(tacc + c * 32, v);
          if (row < brows) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              const int col = c * 32 + j;
              if (col < D)
                *reinterpret_cast<float4*>(brow + col) =
                    make_float4(v[j] * s, v[j + 1] * s, v[j + 2] * s, v[j + 3] * s);
            }
          }
        }
      } else {
        // DP == 128: A in columns [0,128), B in [128,256), TMEM row = matrix row.
        // DP == 64 : one 64-column accumulator; rows 0..63 = A, rows 64..127 = B.
        const bool is_a = (DP == 128) ? true : (row < 64);
        const int mrow = (DP == 128) ? row : (row & 63);
        const float s2 = fa;
#pragma unroll 1
        for (int part = 0; part < (DP == 128 ? 2 : 1); ++part) {
          const bool a_part = (DP == 128) ? (part == 0) : is_a;
          const uint32_t col0 = (DP == 128) ? part * 128 : 0;
#pragma unroll 1
          for (int c = 0; c < DP / 32; ++c) {
            tmem_ld32(tacc + col0 + c * 32, v);
            if (mrow < D) {
              if (a_part) {
                __nv_bfloat16* arow = A_ws + (ws * D + mrow) * D;
#pragma unroll
                for (int j = 0; j < 32; j += 8) {
                  const int col = c * 32 + j;
                  if (col < D) {
                    uint4 pk;
                    pk.x = pack_bf16x2(v[j] * s2, v[j + 1] * s2);
                    pk.y = pack_bf16x2(v[j + 2] * s2, v[j + 3] * s2);
                    pk.z = pack_bf16x2(v[j + 4] * s2, v[j + 5] * s2);
                    pk.w = pack_bf16x2(v[j + 6] * s2, v[j + 7] * s2);
                    *reinterpret_cast<uint4*>(arow + col) = pk;
                  }
                }
              } else {
                float* bmat = B_ws + ws * D * D;
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                  const int col = c * 32 + j;
                  if (col < D) {
                    const long off = kB4 ? b4_index(mrow, col, D) : static_cast<long>(mrow) * D + col;
                    *reinterpret_cast<float4*>(bmat + off) =
                        make_float4(v[j] * fb, v[j + 1] * fb, v[j + 2] * fb, v[j + 3] * fb);
                  }
                }
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
      if constexpr (kFused) {
        // hand the item to the publisher: every epilogue thread's stores (the chain reads them
        // by TMA and cp.async), then one arrival per warp on the slot's barrier
        const int ps = li & 7;
        if (li >= 8 && !mbar_wait(&pub_empty[ps], ((li >> 3) & 1) ^ 1)) {
          give_up(hf, abort_flag);
          break;
        }
        if (leader)
          pub_ids[ps] = (it.bh == 0 && it.t == hf.withhold)
                            ? -1  // test hook: never published
                            : static_cast<int>(static_cast<long>(it.bh) * p.T + it.t);
        fence_async_global();
        __syncwarp();
        if (lane == 0) mbar_arrive(&pub_full[ps]);
      }
    }

  } else if (kFused && warp == kPubWarp) {
    // ---------------------------------------------------------------- publisher (fused)
    // Releases each finished item's stats_flag at GPU scope: the epilogue threads' stores
    // happen-before their arrivals on the slot's barrier, which this thread acquires, and the
    // release makes them visible to the chain (which fences the async proxy after its acquire).
    if (lane == 0) {
      for (int li = 0;; ++li) {
        const int ps = li & 7;
        if (!mbar_wait(&pub_full[ps], (li >> 3) & 1)) {
          if (*abort_flag) break;  // the epilogue gave up: nothing more will arrive
          give_up(hf, abort_flag);
          break;
        }
        const int id = pub_ids[ps];
        if (id == -2) break;
        if (id >= 0) st_release(hf.stats_flag + id, 1);
        mbar_arrive(&pub_empty[ps]);
      }
    }
    __syncwarp();
  } else if (L::kTransform && warp < 6 + L::kTransformThreads / 32) {
    // (the fused kernel's stats CTAs have more warps: the rest stay idle)
    if constexpr (kRope) {
      // ---------------------------------------------------------------- RoPE of the K tiles
      const int tid = threadIdx.x - 192;
      int stage = 0;
      uint32_t phase = 0;
      for (int li = 0;; ++li) {
        const long item = consumer_item(li);
        if (item < 0) break;
        const int t = stats_item<kFused>(item, p, hf, fpb).t;
        bool ok = true;
        for (int tile = 0; tile < n_tiles; ++tile) {
          if (!mbar_wait(&full[stage], phase)) {
            ok = false;
            break;
          }
          const int n0 = tile * kRowsPerTile;
          rope_rotate_tile<DP>(smem + stage * L::kStageBytes, tid, L::kTransformThreads,
                               min(kRowsPerTile, p.N - n0), n0, t, p.D, p.rope, rope_rc);
          fence_async_smem();
          mbar_arrive(&ready[stage]);
          if (++stage == L::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) {
          give_up(hf, abort_flag);
          break;
        }
      }
    } else if constexpr (kLA) {
      // ---------------------------------------------------------------- LA transform warps
      const int tid = threadIdx.x - 192;  // 0..127
      int stage = 0;
      uint32_t phase = 0;
      const int D = p.D;
      for (int li = 0;; ++li) {
        const long item = consumer_item(li);
        if (item < 0) break;
        const int nf = stats_item<kFused>(item, p, hf, fpb).nf;
        bool ok = true;
        for (int tile = 0; tile < item_tiles(nf); ++tile) {
          if (!mbar_wait(&full[stage], phase)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + stage * L::kStageBytes;
          // relu over the K tile's token rows (elementwise, so the swizzle does not matter);
          // rows past the block's last token hold other blocks' keys (or zero fill past the
          // tensor) and are zeroed, so they add nothing to the block's sums
          const __nv_bfloat162 zero2 = __floats2bfloat162_rn(0.f, 0.f);
          const int valid = min(kRowsPerTile, nf * p.N - tile * kRowsPerTile);
#pragma unroll 1
          for (int kb = 0; kb < L::kOpBytes / kBoxBytes; ++kb) {
            // the thread's 8 chunks of the box (8 x 16 B per 128-byte row, rows tid / 8 + 16 u):
            // all loads issued before the first store
            uint4* kt = reinterpret_cast<uint4*>(st + kb * kBoxBytes);
            uint4 x[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) x[u] = kt[tid + 128 * u];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int i = tid + 128 * u;
              __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&x[u]);
#pragma unroll
              for (int j = 0; j < 4; ++j) h2[j] = __hmax2(h2[j], zero2);
              kt[i] = (i >> 3) < valid ? x[u] : make_uint4(0u, 0u, 0u, 0u);
            }
          }
          // ones column at index D of every V row (token), for the normaliser
          *reinterpret_cast<__nv_bfloat16*>(st + L::kOpBytes +
                                            swz128_offset_bf16(tid, D, kBoxBytes)) =
              __float2bfloat16(1.0f);
          fence_async_smem();
          mbar_arrive(&ready[stage]);
          if (++stage == L::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) {
          give_up(hf, abort_flag);
          break;
        }
      }
    }

  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

// A_ws: [B*H*T, D, D] bf16 (GDN only). B_ws: [B*H*T, brows, D] f32, brows = D (GDN) or D+1 (LA),
// row-major, or (kB4, GDN) each D x D matrix in the b4_index layout.
template <int DP, bool kLA, bool kB4, bool kF8 = false, bool kRope = false>
__global__ void __launch_bounds__(StatsLayout<DP, kLA, kF8, kRope>::kThreads, 1)
    gdn_stats_kernel(const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, __nv_bfloat16* __restrict__ A_ws,
                     float* __restrict__ B_ws, Problem p, int frames_per_item) {
  extern __shared__ uint8_t smem_raw[];
  const Handoff none{nullptr, nullptr, nullptr, nullptr, nullptr, 1, 1, -1, 0, 0};
  stats_body<DP, kLA, false, kB4, kF8, kRope>(&tm_k, &tm_v, A_ws, B_ws, p, none,
                                              align1k(smem_raw), frames_per_item);
}

}  // namespace gdn
