// Output: O_t = Q_t S_t^T for every frame of every head, in parallel (every token of frame t
// reads the post-update state S_t, so attention is bidirectional inside a frame and causal
// across frames).
//
// Per work item (b, t, h): S_t is loaded once as a K-major B operand -- for GDN one contiguous
// bulk copy of the DP x DP bf16 block in the core-matrix layout of s8_offset_bytes (the chain's
// output), for LA a TMA load of the row-major (D+1) x D state; the frame's Q rows stream through a ring of 128-token TMA tiles (K-major A
// operand); each tile is one 128 x DP x DP tcgen05 GEMM into a double-buffered TMEM
// accumulator; the epilogue converts rows to bf16 into a 128B-swizzled staging tile in shared
// memory and one thread TMA-stores it to out[b, t, n, h, :] (rows past N and columns past D are
// clipped by the tensor map), so global writes are whole coalesced lines.
//
// LA mode (block-causal linear attention): Q tiles are passed through relu in shared memory
// by 4 transform warps before the MMA, the state row D holds the normaliser z, and the
// epilogue divides the first D columns by (column D + 1e-6).
// fp8 mode (e4m3 Q, DP = 128): the Q tile is TMA-loaded into the second box of its bf16 stage,
// the 4 transform warps convert it in place (exactly), and the epilogue multiplies by the
// frame's Q scale.
// RoPE mode (the fused 3D rotary prologue): 4 * DP/64 transform warps rotate each Q tile in
// place (one 64-dim box of one token row per thread) before the MMA.
//
// Warp roles: warp 0 TMA producer, warp 1 TMEM allocator + MMA issuer, warps 2 .. 2+4G-1
// epilogue (G column groups of 4 warps; warp w reads TMEM lanes 32*(w%4) and DP/G columns), then
// (LA only) 4 transform warps. The epilogue sets the pace of a tile (TMEM read-out, bf16
// conversion, staging): with G = 1 a tile took about 1.7 us per SM, under the HBM share.
//
// Standalone (gdn_output_kernel): GDN work item i = (b*T + t)*H + h, S_t at workspace row
// (b*H+h)*T + t; LA work item i = (b*n_blocks + j)*H + h, a block of frames over the flattened
// token rows, its state at row (b*H+h)*n_blocks + j.
// Fused (output role of gdn_fused_kernel): work item i = t*B*H + b*H + h, taken in the order the
// chains published them (a queue the chain CTAs append to), S_t loaded from ring row
// (b*H+h)*Rs + t%Rs (chain_prog is checked again); out_flag releases the slot as soon as S_t
// is in shared memory.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "rope_kernel.cuh"

namespace gdn {

// With RoPE at DP = 128 the layout gives up a Q stage for the table copy of rope_stage_rc (the
// 720p clip: 4.53 ms against 4.76 with three stages and the table read through L1, 5.06 with
// three stages and one state buffer).
#ifndef GDN_ROPE_OUT_SBUFS
#define GDN_ROPE_OUT_SBUFS 2
#endif
#ifndef GDN_ROPE_OUT_QSTAGES
#define GDN_ROPE_OUT_QSTAGES 2
#endif
#ifndef GDN_ROPE_OUT_OBUFS
#define GDN_ROPE_OUT_OBUFS 2
#endif
// fp8 inputs at DP = 128: Q stages and output staging tiles (the 720p clip: 2.31 ms with 3 and
// 2, 2.63 with 4 and 1, 2.87 with 2 and 3; the role needs its stores in flight as much as its
// loads)
#ifndef GDN_F8_OUT_QSTAGES
#define GDN_F8_OUT_QSTAGES 3
#endif
#ifndef GDN_F8_OUT_OBUFS
#define GDN_F8_OUT_OBUFS 2
#endif

// e4m3_row_to_bf16_tile (the in-place conversion of an fp8 Q tile into the bf16 operand layout)
// with explicit shared-space loads and stores on the tile's 32-bit shared address: every lane
// of the warp reads its chunks before any lane writes, as there.
template <int kParts>
__device__ __forceinline__ void e4m3_row_to_bf16_tile_s(uint32_t tile, int row, int part) {
  static_assert(kParts == 1 || kParts == 2 || kParts == 4, "parts of a row");
  constexpr int kC = 8 / kParts;
  const uint32_t b0 = tile + row * 128;
  const uint32_t b1 = tile + 16384 + row * 128;
  const uint32_t sw = row & 7;
  uint4 in[kC];
#pragma unroll
  for (int i = 0; i < kC; ++i) in[i] = rope_lds128(b1 + (((part * kC + i) ^ sw) << 4));
  if (kParts > 1) __syncwarp();
#pragma unroll
  for (int i = 0; i < kC; ++i) {
    // fp8 chunk c = dims 16c..16c+15 -> bf16 chunks 2c, 2c+1 of the 16 chunks of 8 dims
    const int c = part * kC + i;
    uint4 lo, hi;
    e4m3x16_to_bf16(in[i], lo, hi);
    const int k0 = 2 * c, k1 = 2 * c + 1;  // 8-dim chunk index over 128 dims
    rope_sts128((k0 < 8 ? b0 : b1) + (((k0 & 7) ^ sw) << 4), lo);
    rope_sts128((k1 < 8 ? b0 : b1) + (((k1 & 7) ^ sw) << 4), hi);
  }
}

// kRopeGroups: groups of 128 threads (4 warps) in the RoPE transform of the Q tiles.
template <int DP, bool kLA, int kG = 4, bool kF8 = false, bool kRope = false,
          int kRopeGroups = DP / 64>
struct OutputLayout {
  static_assert(!kF8 || (DP == 128 && !kLA), "fp8 inputs: DP = 128, GDN only");
  static_assert(!kRope || (!kF8 && !kLA), "RoPE prologue: bf16 GDN only");
  static constexpr bool kTransform = kLA || kF8 || kRope;
  // transform warps: 4 (one token row each; fp8: kF8Parts lanes per row), or for RoPE 4 per group
  static constexpr int kF8Parts = 2;  // fp8: lanes per Q row in the e4m3 -> bf16 conversion
  static constexpr int kXfWarps = kRope ? 4 * kRopeGroups : (kF8 ? 4 * kF8Parts : 4);
  static constexpr int kEpiWarps = 4 * kG;
  static constexpr int kCols = DP / kG;                // columns per epilogue thread
  static constexpr int kChunk = kCols < 32 ? kCols : 32;
  static constexpr int kBoxes = DP / 64;
  static constexpr int kQBytes = kBoxes * kBoxBytes;   // 128 tokens x DP bf16
  static constexpr int kSBufBytes = DP * DP * 2;       // DP/64 blocks of DP rows x 128 B
  // state buffers: items in flight past the state load (the fused role waits on the chain, so
  // more of them hide its hand-off latency; DP = 128 has no shared memory left for more)
  static constexpr int kSBufs = (DP == 128) ? (kRope ? GDN_ROPE_OUT_SBUFS : 2) : 4;
  static constexpr int kStages =
      (DP == 128) ? (kRope ? GDN_ROPE_OUT_QSTAGES : (kF8 ? GDN_F8_OUT_QSTAGES : 3)) : 8;
  static constexpr int kTabBytes = kRope ? kRopeSmemTabBytes : 0;
  static constexpr int kThreads = (2 + kEpiWarps + (kTransform ? kXfWarps : 0)) * 32;
  static constexpr int kQLoadBytes = kF8 ? kQBytes / 2 : kQBytes;  // TMA bytes per Q tile
  static constexpr int kTmemCols = (2 * DP < 32) ? 32 : 2 * DP;
  static constexpr int kOBytes = kQBytes;  // one bf16 output tile
  static constexpr int kOBufs =  // staging tiles
      DP == 128 ? (kRope ? GDN_ROPE_OUT_OBUFS : (kF8 ? GDN_F8_OUT_OBUFS : 2)) : 2;
  static constexpr int kBarrierBytes = 1024;
  static constexpr int kSmemBytes =
      kSBufs * kSBufBytes + kStages * kQBytes + kOBufs * kOBytes + kBarrierBytes + kTabBytes + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
  // barriers, item ring, TMEM slot and the fused publisher's ring within kBarrierBytes
  static_assert(8 * (3 * kStages + 2 * kSBufs + 4 + 8 + 1) + 32 + 8 + 8 * 16 + 32 <= kBarrierBytes,
                "barriers");
};

struct OutputItem {
  int h, bt, bh, t;
  int n_tiles;  // 128-row tiles of the item
  int rows;     // token rows of the item (LA: all frames of its block)
  int row0;     // LA: first row in the flattened (b, t, n) token space of the 3-D maps
  long srow;    // LA: row of the block's state
};

// GDN items are frames (b, t, h); LA items are blocks (b, j, h) of F frames, whose N*F rows are
// contiguous in the flattened token space, so their tiles span frames (10 tiles of 128 rows for
// 3 frames of 390 tokens instead of 3 x 4).
template <bool kFused, bool kLA = false>
__device__ __forceinline__ OutputItem output_item(long item, const Problem& p, int F = 1) {
  OutputItem it;
  it.rows = p.N;
  it.row0 = 0;
  it.srow = 0;
  if constexpr (kLA) {
    const int nblk = (p.T + F - 1) / F;
    it.h = static_cast<int>(item % p.H);
    const int bj = static_cast<int>(item / p.H);
    const int b = bj / nblk;
    const int j = bj - b * nblk;
    it.t = j * F;
    it.bt = b * p.T + it.t;
    it.bh = b * p.H + it.h;
    it.rows = min(F, p.T - it.t) * p.N;
    it.row0 = it.bt * p.N;
    it.srow = static_cast<long>(it.bh) * nblk + j;
  } else if constexpr (kFused) {
    const int BH = p.B * p.H;
    it.t = static_cast<int>(item / BH);
    it.bh = static_cast<int>(item - static_cast<long>(it.t) * BH);
    const int b = it.bh / p.H;
    it.h = it.bh - b * p.H;
    it.bt = b * p.T + it.t;
  } else {
    it.h = static_cast<int>(item % p.H);
    it.bt = static_cast<int>(item / p.H);
    const int b = it.bt / p.T;
    it.t = it.bt - b * p.T;
    it.bh = b * p.H + it.h;
  }
  it.n_tiles = (it.rows + kRowsPerTile - 1) / kRowsPerTile;
  return it;
}

// frames_per_block: 1 for GDN (frame t reads S_t); F for LA (frame t reads the state at the end
// of its block of F frames). GDN states come from S_src (DP*DP bf16 per row, s8 layout); LA
// states through tm_s.
// LA: tm_q and tm_o are 3-D maps over the flattened token rows, and out (the raw output) takes
// the row stores of a block's last, partial tile (a 128-row TMA store would also overwrite the
// first rows of the next block, which another CTA writes).
template <int DP, bool kLA, bool kFused, int kG, bool kF8 = false, bool kRope = false,
          int kRopeGroups = DP / 64>
__device__ __forceinline__ void output_body(const CUtensorMap* tm_q, const CUtensorMap* tm_s,
                                            const __nv_bfloat16* __restrict__ S_src,
                                            const CUtensorMap* tm_o, const Problem& p,
                                            int frames_per_block, const Handoff& hf,
                                            uint8_t* smem, __nv_bfloat16* out = nullptr) {
  using L = OutputLayout<DP, kLA, kG, kF8, kRope, kRopeGroups>;
  constexpr int kEpiThreads = 32 * L::kEpiWarps;
  uint8_t* s_buf = smem;                                  // kSBufs state buffers
  uint8_t* q_ring = smem + L::kSBufs * L::kSBufBytes;     // kStages Q tiles
  uint8_t* o_stage = q_ring + L::kStages * L::kQBytes;  // kOBufs output staging tiles
  uint64_t* full = reinterpret_cast<uint64_t*>(o_stage + L::kOBufs * L::kOBytes);
  uint64_t* ready = full + L::kStages;
  uint64_t* empty = ready + L::kStages;
  uint64_t* s_full = empty + L::kStages;
  uint64_t* s_empty = s_full + L::kSBufs;
  uint64_t* acc_full = s_empty + L::kSBufs;
  uint64_t* acc_empty = acc_full + 2;
  ItemRing ring{reinterpret_cast<int*>(acc_empty + 2 + 9), acc_empty + 2};  // fused only
  uint64_t* mma_drain = acc_empty + 2 + 8;  // all of this CTA's MMAs are complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ring.ids + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // fused: the MMA warp hands each item's "S_t is in shared memory" to the publisher warp through
  // an 8-slot ring, so the GPU-scope release of out_flag does not hold up the MMA issue
  uint64_t* pub_full = reinterpret_cast<uint64_t*>(tmem_slot + 2);
  uint64_t* pub_empty = pub_full + 8;
  int* pub_ids = reinterpret_cast<int*>(pub_empty + 8);
  constexpr uint32_t kPubWarp = 18;  // the fused CTA's last warp (idle in the output role)

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int F = frames_per_block;
  const long n_items = static_cast<long>(p.B) * (kLA ? (p.T + F - 1) / F : p.T) * p.H;
  const long cta0 = kFused ? blockIdx.x - hf.base : blockIdx.x;
  const long ncta = kFused ? hf.count : gridDim.x;
  // item li of this CTA: standalone a static stride, fused the role's work counter. Returns -1
  // when there are no more items, -2 on a timed-out wait.
  auto producer_item = [&](int li) -> long {
    if constexpr (kFused)
      return ring.produce_queued(li, hf.next_item, hf.ready_items, n_items, hf.abort);
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
      mbar_init(&ready[s], 32 * L::kXfWarps);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < L::kSBufs; ++a) {
      mbar_init(&s_full[a], 1);
      mbar_init(&s_empty[a], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], kEpiThreads);
    }
    for (int i = 0; i < 8; ++i) mbar_init(&ring.bars[i], 1);
    mbar_init(mma_drain, 1);
    for (int i = 0; i < 8; ++i) {
      mbar_init(&pub_full[i], 1);
      mbar_init(&pub_empty[i], 1);
    }
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
    rope_rc = rope_stage_rc(reinterpret_cast<float2*>(o_stage + L::kOBufs * L::kOBytes + L::kBarrierBytes),
                            p.rope, threadIdx.x, blockDim.x);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (elect_one()) {
      tma_prefetch_desc(tm_q);
      if constexpr (kLA) tma_prefetch_desc(tm_s);
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_state = policy_evict_last();
      StageFills<L::kStages> fills;
      StageFills<L::kSBufs> s_fills;
      int stage = 0;
      uint32_t phase = 0;
      // Q tile `tile` of item `it` into the next stage; false if the wait for the stage ran out
      auto load_q = [&](const OutputItem& it, int tile) -> bool {
        if (!mbar_wait(&empty[stage], phase ^ 1)) return false;
        mbar_arrive_expect_tx(&full[stage], L::kQLoadBytes);
        if constexpr (kLA) {
          // 128 flattened token rows (they may run into the next frame of the block)
#pragma unroll
          for (int kb = 0; kb < L::kBoxes; ++kb)
            tma_load_3d(q_ring + stage * L::kQBytes + kb * kBoxBytes, tm_q, &full[stage],
                        kb * 64, it.h, it.row0 + tile * kRowsPerTile, pol_stream);
        } else if constexpr (kF8) {
          // one 128-byte-wide e4m3 box, into the stage's second bf16 box
          tma_load_4d(q_ring + stage * L::kQBytes + kBoxBytes, tm_q, &full[stage], 0, it.h,
                      tile * kRowsPerTile, it.bt, pol_stream);
        } else {
#pragma unroll
          for (int kb = 0; kb < L::kBoxes; ++kb)
            tma_load_4d(q_ring + stage * L::kQBytes + kb * kBoxBytes, tm_q, &full[stage],
                        kb * 64, it.h, tile * kRowsPerTile, it.bt, pol_stream);
        }
        fills.filled(stage, phase);
        if (++stage == L::kStages) {
          stage = 0;
          phase ^= 1;
        }
        return true;
      };
      for (int li = 0; !*abort_flag; ++li) {
        const long item = producer_item(li);
        if (item < 0) break;
        const OutputItem it = output_item<kFused, kLA>(item, p, F);
        int srow;
        if constexpr (kFused) {
          srow = it.bh * hf.Rs + it.t % hf.Rs;
        } else {
          // GDN: the frame's own state (F = 1); LA: the state after the frame's block
          const int n_blocks = (p.T + F - 1) / F;
          srow = it.bh * n_blocks + it.t / F;
        }
        const int sb = li % L::kSBufs;
        const uint32_t sph = (li / L::kSBufs) & 1;
        if (!mbar_wait(&s_empty[sb], sph ^ 1)) {
          give_up(hf, abort_flag);
          break;
        }
        if constexpr (kFused) {
          if (!wait_flag_ge(hf.chain_prog + it.bh, it.t + 1, hf.abort)) {
            give_up(hf, abort_flag);
            break;
          }
          fence_async_global();
        }
        mbar_arrive_expect_tx(&s_full[sb], L::kSBufBytes);
        if constexpr (kLA) {
#pragma unroll
          for (int kb = 0; kb < L::kBoxes; ++kb)
            tma_load_3d(s_buf + sb * L::kSBufBytes + kb * DP * 128, tm_s, &s_full[sb], kb * 64,
                        0, srow, pol_state);
        } else {
          bulk_load(s_buf + sb * L::kSBufBytes, S_src + static_cast<long>(srow) * DP * DP,
                    L::kSBufBytes, &s_full[sb], pol_state);
        }
        s_fills.filled(sb, sph);
        bool ok = true;
        for (int tile = 0; ok && tile < it.n_tiles; ++tile) ok = load_q(it, tile);
        if (!ok) {
          give_up(hf, abort_flag);
          break;
        }
      }
      // this thread's copies have landed, whatever the exit path
      fills.drain(full);
      s_fills.drain(s_full);
    }
  } else if (warp == 1) {
    constexpr uint32_t idesc = idesc_bf16(128, DP, false, false);
    int stage = 0;
    uint32_t phase = 0;
    int tc = 0;  // tiles processed (accumulator ring position)
    bool ok = true;
    // fused: hand item li's out_flag (id >= 0) or the end (-2) to the publisher
    auto hand_off = [&](int li, int id) -> bool {
      const int ps = li & 7;
      if (li >= 8 && !mbar_wait(&pub_empty[ps], ((li >> 3) & 1) ^ 1)) return false;
      if (lane == 0) {
        pub_ids[ps] = id;
        mbar_arrive(&pub_full[ps]);
      }
      __syncwarp();
      return true;
    };
    for (int li = 0; ok; ++li) {
      const long item = consumer_item(li);
      if (item == -2) ok = false;
      if (item < 0) {
        if constexpr (kFused)
          if (ok && !hand_off(li, -2)) ok = false;
        break;
      }
      const int sb = li % L::kSBufs;
      if (!mbar_wait(&s_full[sb], (li / L::kSBufs) & 1)) {
        ok = false;
        break;
      }
      const OutputItem it = output_item<kFused, kLA>(item, p, F);
      if constexpr (kFused) {
        // S_t is in shared memory: its ring slot may be overwritten by the chain
        if (!hand_off(li, static_cast<int>(static_cast<long>(it.bh) * p.T + it.t))) {
          ok = false;
          break;
        }
      }
      const uint32_t s_base = smem_u32(s_buf + sb * L::kSBufBytes);
      for (int tile = 0; tile < it.n_tiles; ++tile, ++tc) {
        const int acc = tc & 1;
        if (!mbar_wait(&acc_empty[acc], ((tc >> 1) & 1) ^ 1) ||
            !mbar_wait(L::kTransform ? &ready[stage] : &full[stage], phase)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const uint32_t q_base = smem_u32(q_ring + stage * L::kQBytes);
#pragma unroll
          for (int ks = 0; ks < DP / 16; ++ks) {
            const uint64_t da =
                smem_desc(q_base + (ks >> 2) * kBoxBytes + (ks & 3) * 32, 16, 1024);
            // LA: row-major state through a 128B-swizzled TMA box; GDN: core matrices, key
            // groups 2ks and 2ks+1 (DP*16 bytes apart), 8-row groups 128 bytes apart
            const uint64_t db =
                kLA ? smem_desc(s_base + (ks >> 2) * DP * 128 + (ks & 3) * 32, 16, 1024)
                    : smem_desc_noswz(s_base + ks * 2 * DP * 16, DP * 16, 128);
            mma_bf16(tmem_base + acc * DP, da, db, idesc, ks != 0);
          }
          mma_commit(&empty[stage]);
          mma_commit(&acc_full[acc]);
        }
        __syncwarp();
        if (++stage == L::kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      if (elect_one()) mma_commit(&s_empty[sb]);
      __syncwarp();
    }
    if (!ok) give_up(hf, abort_flag);
    // every MMA issued here has completed before TMEM is released
    if (elect_one()) mma_commit(mma_drain);
    __syncwarp();
    mbar_wait(mma_drain, 0);
  } else if (warp < 2 + L::kEpiWarps) {
    // ---------------------------------------------------------------- epilogue
    const uint32_t quarter = warp & 3;
    const int c0 = ((warp - 2) >> 2) * L::kCols;  // first column of this warp's group
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem_base + ((quarter * 32) << 16);
    const int D = p.D;
    const bool leader = (threadIdx.x == 64);
    const uint64_t pol_out = policy_evict_first();
    if (leader) tma_prefetch_desc(tm_o);
    int tc = 0;
    bool ok = true;
    for (int li = 0; ok; ++li) {
      const long item = consumer_item(li);
      bool lost = item == -2;
      if constexpr (kFused) lost = named_bar_any(1, kEpiThreads, lost);  // uniform across the epilogue
      if (lost) ok = false;
      if (lost || item < 0) break;
      const OutputItem it = output_item<kFused, kLA>(item, p, F);
      for (int tile = 0; tile < it.n_tiles; ++tile, ++tc) {
        const int acc = tc & 1;
        const int valid = min(kRowsPerTile, it.rows - tile * kRowsPerTile);
        // LA: a block's last tile runs into the next block's rows, so its valid rows are stored
        // row by row instead of through the TMA box
        const bool row_stores = kLA && valid < kRowsPerTile;
        const bool waited = mbar_wait(&acc_full[acc], (tc >> 1) & 1);
        // staging buffer tc % kOBufs is free once the store issued kOBufs tiles ago has read it
        if (leader) bulk_wait_read<L::kOBufs - 1>();
        if (named_bar_any(1, kEpiThreads, !waited)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // warps whose 32 rows are all past the item's last token skip the read-out: the TMA
        // store clips at N (GDN), and LA stores such tiles row by row
        uint8_t* ob = o_stage + (tc % L::kOBufs) * L::kOBytes;
        if (static_cast<int>(quarter) * 32 < valid) {
          const uint32_t tacc = lane_base + acc * DP;
          float scale = 1.f;
          if constexpr (kLA) scale = 1.f / (tmem_ld1(tacc + D) + 1e-6f);  // normaliser, column D
          if constexpr (kF8) scale = __ldg(p.q_scale + static_cast<long>(it.bt) * p.H + it.h);
          float v[L::kChunk];
#pragma unroll 1
          for (int c = c0; c < c0 + L::kCols; c += L::kChunk) {
            if constexpr (L::kChunk == 32)
              tmem_ld32(tacc + c, v);
            else
              tmem_ld16(tacc + c, v);
#pragma unroll
            for (int j = 0; j < L::kChunk; j += 8) {
              uint4 pk;
              pk.x = pack_bf16x2(v[j] * scale, v[j + 1] * scale);
              pk.y = pack_bf16x2(v[j + 2] * scale, v[j + 3] * scale);
              pk.z = pack_bf16x2(v[j + 4] * scale, v[j + 5] * scale);
              pk.w = pack_bf16x2(v[j + 6] * scale, v[j + 7] * scale);
              if (row_stores) {
                if (row < valid && c + j < D)
                  *reinterpret_cast<uint4*>(
                      out + (static_cast<long>(it.row0 + tile * kRowsPerTile + row) * p.H + it.h) *
                                D + c + j) = pk;
              } else {
                *reinterpret_cast<uint4*>(ob + swz128_offset_bf16(row, c + j, kBoxBytes)) = pk;
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[acc]);
        fence_async_smem();
        named_bar(1, kEpiThreads);
        if (leader) {
          if (!row_stores) {
#pragma unroll
            for (int kb = 0; kb < L::kBoxes; ++kb) {
              if constexpr (kLA)
                tma_store_3d(tm_o, ob + kb * kBoxBytes, kb * 64, it.h,
                             it.row0 + tile * kRowsPerTile, pol_out);
              else
                tma_store_4d(tm_o, ob + kb * kBoxBytes, kb * 64, it.h, tile * kRowsPerTile,
                             it.bt, pol_out);
            }
          }
          // one bulk group per tile, empty for a tile stored row by row, so that the wait for
          // "the store issued kOBufs tiles ago has read its staging buffer" counts tiles: without
          // it, after an LA block's row-stored last tile the next tile's epilogue could overwrite
          // the staging buffer a still-pending store was reading
          bulk_commit();
        }
      }
    }
    if (leader) bulk_wait_all();
    if (!ok) give_up(hf, abort_flag);
  } else if (kFused && warp == kPubWarp) {
    // ---------------------------------------------------------------- publisher (fused)
    // Releases out_flag of each item whose S_t the MMA warp has seen land in shared memory
    // (the bulk copy completed on s_full before the hand-off), at GPU scope.
    if (lane == 0) {
      for (int li = 0;; ++li) {
        const int ps = li & 7;
        if (!mbar_wait(&pub_full[ps], (li >> 3) & 1)) {
          if (*abort_flag) break;  // the MMA warp gave up: nothing more will arrive
          give_up(hf, abort_flag);
          break;
        }
        const int id = pub_ids[ps];
        if (id == -2) break;
        st_release(hf.out_flag + id, 1);
        mbar_arrive(&pub_empty[ps]);
      }
    }
    __syncwarp();
  } else if (L::kTransform && warp < 2 + L::kEpiWarps + L::kXfWarps) {
    // (the fused kernel's output CTAs have more warps: the rest stay idle)
    if constexpr (kRope) {
      // ---------------------------------------------------------------- RoPE of the Q tiles
      const int tid = threadIdx.x - 32 * (2 + L::kEpiWarps);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int li = 0; ok; ++li) {
        const long item = consumer_item(li);
        if (item < 0) break;
        const OutputItem it = output_item<kFused, kLA>(item, p, F);
        for (int tile = 0; tile < it.n_tiles; ++tile) {
          if (!mbar_wait(&full[stage], phase)) {
            ok = false;
            break;
          }
          const int n0 = tile * kRowsPerTile;
          rope_rotate_tile<DP>(q_ring + stage * L::kQBytes, tid, 32 * L::kXfWarps,
                               min(kRowsPerTile, p.N - n0), n0, it.t, p.D, p.rope, rope_rc);
          fence_async_smem();
          mbar_arrive(&ready[stage]);
          if (++stage == L::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) give_up(hf, abort_flag);
    } else if constexpr (kF8) {
      // ---------------------------------------------------------------- e4m3 Q conversion
      const int tid = threadIdx.x - 32 * (2 + L::kEpiWarps);  // row tid / kF8Parts, its part
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int li = 0; ok; ++li) {
        const long item = consumer_item(li);
        if (item < 0) break;
        const int n_tiles = output_item<kFused, kLA>(item, p, F).n_tiles;
        for (int tile = 0; tile < n_tiles; ++tile) {
          if (!mbar_wait(&full[stage], phase)) {
            ok = false;
            break;
          }
          e4m3_row_to_bf16_tile_s<L::kF8Parts>(smem_u32(q_ring + stage * L::kQBytes),
                                               tid / L::kF8Parts, tid % L::kF8Parts);
          fence_async_smem();
          mbar_arrive(&ready[stage]);
          if (++stage == L::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) give_up(hf, abort_flag);
    } else if constexpr (kLA) {
      // ---------------------------------------------------------------- relu(Q) transform
      const int tid = threadIdx.x - 32 * (2 + L::kEpiWarps);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int li = 0; ok; ++li) {
        const long item = consumer_item(li);
        if (item < 0) break;
        const OutputItem it = output_item<kFused, kLA>(item, p, F);
        for (int tile = 0; tile < it.n_tiles; ++tile) {
          if (!mbar_wait(&full[stage], phase)) {
            ok = false;
            break;
          }
          const __nv_bfloat162 zero2 = __floats2bfloat162_rn(0.f, 0.f);
          // rows past the block's last token belong to other blocks: their outputs are not
          // stored, so they need no relu
          const int valid = min(kRowsPerTile, it.rows - tile * kRowsPerTile);
#pragma unroll 1
          for (int kb = 0; kb < L::kBoxes; ++kb) {
            // the thread's 8 chunks of the box (8 x 16 B per 128-byte box row, rows tid / 8 +
            // 16 u): all loads issued before the first store
            uint4* qt = reinterpret_cast<uint4*>(q_ring + stage * L::kQBytes + kb * kBoxBytes);
            uint4 x[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
              if (((tid + 128 * u) >> 3) < valid) x[u] = qt[tid + 128 * u];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              if (((tid + 128 * u) >> 3) >= valid) continue;
              __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&x[u]);
#pragma unroll
              for (int j = 0; j < 4; ++j) h2[j] = __hmax2(h2[j], zero2);
              qt[tid + 128 * u] = x[u];
            }
          }
          fence_async_smem();
          mbar_arrive(&ready[stage]);
          if (++stage == L::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) give_up(hf, abort_flag);
    }

  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

template <int DP, bool kLA, bool kF8 = false, bool kRope = false>
__global__ void __launch_bounds__(OutputLayout<DP, kLA, 4, kF8, kRope>::kThreads, 1)
    gdn_output_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_s,
                      const __nv_bfloat16* __restrict__ S_src,
                      const __grid_constant__ CUtensorMap tm_o, Problem p, int frames_per_block,
                      __nv_bfloat16* out) {
  extern __shared__ uint8_t smem_raw[];
  const Handoff none{nullptr, nullptr, nullptr, nullptr, nullptr, 1, 1, -1, 0, 0};
  output_body<DP, kLA, false, 4, kF8, kRope>(&tm_q, &tm_s, S_src, &tm_o, p, frames_per_block,
                                             none, align1k(smem_raw), out);
}

}  // namespace gdn
