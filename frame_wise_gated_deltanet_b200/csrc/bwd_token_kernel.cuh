// Token-side gradient GEMMs of the backward, every frame of every head in parallel. Per frame
// (b, t, h) and 128-token tile, one accumulator sums kTerms products X_i Y_i^(T) of a token
// tile X_i (TMA, 128B swizzle, K-major) and a frame matrix Y_i (bf16 DP x DP in the s8 layout,
// one bulk copy per frame); the epilogue scales the tile and TMA-stores it as bf16:
//
//   dQ_t = dO_t S_t                      (1 term, Y = S_t read MN-major: contraction over v)
//   dV_t = s beta_t * K_t G_t^T          (1 term, Y = G_t read K-major: contraction over k)
//   dK_t = s beta_t * (V_t G_t + K_t W'_t)   (2 terms: G_t MN-major, W'_t K-major)
//
// kDualV: dK_t and dV_t from one pass (the K tile and G_t are shared): a second accumulator
// takes K_t G_t^T, and the epilogue stores both tiles through one staging buffer.
// kDualE: dQ_t and the output statistic E_t = dO_t^T Q_t from one pass over dO: each stage holds
// a dO tile and a Q tile; dQ_t takes the dO tile K-major as above, and a per-frame accumulator sums
// dO^T Q over the frame's tiles with both read MN-major (the statistics kernel's reduction, in the
// same order); the epilogue writes E_t as f32 in the four-key interleaved layout of b4_index.
//
// with s the key scale, G_t = dL/dS_t from the backward chain and W'_t = -s gamma_t (S_{t-1}^T
// G_t + G_t^T S_{t-1}) from the per-frame kernel (K_t here is the unscaled key tile, so both
// factors of s are in these scalars).
//
// The same pipeline as the forward's output GEMM: warp 0 TMA producer, warp 1 TMEM allocator +
// MMA issuer, warps 2..17 epilogue (4 column groups of 4 warps). One term: two frame-matrix
// buffers, three token stages, two staging tiles. Two terms: one buffer per frame matrix, two
// stages of two token tiles, one staging tile (227 KB of shared memory either way).
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace gdn {

template <int DP, int kTerms, bool kDualV = false, bool kDualE = false>
struct BwdTokenLayout {
  static_assert(DP == 128 && (kTerms == 1 || kTerms == 2), "DP = 128, one or two terms");
  static_assert(!kDualV || kTerms == 2, "the dK/dV pass has two terms");
  static_assert(!kDualE || (kTerms == 2 && !kDualV), "the dQ/E pass has two token tiles");
  static constexpr int kAccs = kDualV ? 2 : 1;  // accumulators per tile
  static constexpr int kEpiWarps = 16;
  static constexpr int kCols = DP / 4;  // columns per epilogue thread
  static constexpr int kBoxes = DP / 64;
  static constexpr int kXBytes = kBoxes * kBoxBytes;  // one 128-token tile
  static constexpr int kYBytes = DP * DP * 2;
  static constexpr int kYPer = kDualE ? 1 : kTerms;  // frame matrices per item
  static constexpr int kYBufs = (kTerms == 1 || kDualE) ? 2 : 1;
  static constexpr int kStages = kTerms == 1 ? 3 : 2;
  static constexpr int kOBufs = kTerms == 1 ? 2 : 1;
  static constexpr int kStageBytes = kTerms * kXBytes;
  static constexpr int kThreads = (2 + kEpiWarps) * 32;
  // tile accumulators (two), then (kDualE) two per-frame E accumulators
  static constexpr int kTmemCols = kDualE ? 4 * DP : 2 * kAccs * DP;
  static constexpr int kOBytes = kXBytes;
  static constexpr int kSmemBytes =
      kYBufs * kYPer * kYBytes + kStages * kStageBytes + kOBufs * kOBytes + 512 + 1024;
};

struct BwdTokenArgs {
  const __nv_bfloat16* Y0;  // frame matrices of term 0 / 1, DP*DP bf16 per row (b*H+h)*T + t
  const __nv_bfloat16* Y1;
  const float* beta;        // non-null: scale by key_scale * beta[b, t, h], else 1
  int t_lo, t_hi;           // the frames [t_lo, t_hi) of every head
  float* E;                 // kDualE: E_t, f32 D x D per row (b*H+h)*T + t (b4_index layout)
};

// kMN0 / kMN1: the term's frame matrix is read MN-major (contraction over its rows).
// kDualV: tm_o2 takes s beta_t * X1 Y0^T (Y0 read K-major) from a second accumulator.
// kDualE: X0 = dO, X1 = Q, one term (X0 Y0 with Y0 = S_t MN-major), and E_t = X0^T X1 into a.E.
template <int DP, int kTerms, bool kMN0, bool kMN1, bool kDualV = false, bool kDualE = false>
__global__ void __launch_bounds__(BwdTokenLayout<DP, kTerms, kDualV, kDualE>::kThreads, 1)
    gdn_bwd_token_kernel(const __grid_constant__ CUtensorMap tm_x0,
                         const __grid_constant__ CUtensorMap tm_x1,
                         const __grid_constant__ CUtensorMap tm_o,
                         const __grid_constant__ CUtensorMap tm_o2, BwdTokenArgs a, Problem p) {
  using L = BwdTokenLayout<DP, kTerms, kDualV, kDualE>;
  constexpr int kAccs = L::kAccs;
  constexpr int kMmaTerms = kDualE ? 1 : kTerms;  // products summed into a tile accumulator
  constexpr int kEpiThreads = 32 * L::kEpiWarps;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1k(smem_raw);
  uint8_t* y_buf = smem;                                     // [kYBufs][kYPer] frame matrices
  uint8_t* x_ring = y_buf + L::kYBufs * L::kYPer * L::kYBytes;  // [kStages][kTerms] token tiles
  uint8_t* o_stage = x_ring + L::kStages * L::kStageBytes;    // [kOBufs] staging tiles
  uint64_t* full = reinterpret_cast<uint64_t*>(o_stage + L::kOBufs * L::kOBytes);
  uint64_t* empty = full + L::kStages;
  uint64_t* y_full = empty + L::kStages;
  uint64_t* y_empty = y_full + 2;
  uint64_t* acc_full = y_empty + 2;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* e_full = acc_empty + 2;  // kDualE: E accumulator of item li % 2 complete / read
  uint64_t* e_empty = e_full + 2;
  uint64_t* mma_drain = e_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int nt = a.t_hi - a.t_lo;
  const long n_items = static_cast<long>(p.B) * nt * p.H;
  const int n_tiles = (p.N + kRowsPerTile - 1) / kRowsPerTile;
  const Handoff none{nullptr, nullptr, nullptr, nullptr, nullptr, 1, 1, -1, 0, 0};
  // item i = (b*nt + t - t_lo)*H + h; bt = b*T + t
  auto decode = [&](long item, int& bt, int& h, long& yrow) {
    h = static_cast<int>(item % p.H);
    const int r = static_cast<int>(item / p.H);
    const int b = r / nt;
    const int t = a.t_lo + (r - b * nt);
    bt = b * p.T + t;
    yrow = (static_cast<long>(b) * p.H + h) * p.T + t;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&y_full[i], 1);
      mbar_init(&y_empty[i], 1);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], kEpiThreads);
      mbar_init(&e_full[i], 1);
      mbar_init(&e_empty[i], kEpiThreads);
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
    // ---------------------------------------------------------------- producer
    if (elect_one()) {
      tma_prefetch_desc(&tm_x0);
      if (kTerms == 2) tma_prefetch_desc(&tm_x1);
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_frame = policy_evict_last();
      StageFills<L::kStages> fills;
      StageFills<2> y_fills;
      int stage = 0;
      uint32_t phase = 0;
      int li = 0;
      for (long item = blockIdx.x; item < n_items && !*abort_flag; item += gridDim.x, ++li) {
        int bt, h;
        long yrow;
        decode(item, bt, h, yrow);
        const int yb = li % L::kYBufs;
        const uint32_t yph = (li / L::kYBufs) & 1;
        if (!mbar_wait(&y_empty[yb], yph ^ 1)) {
          give_up(none, abort_flag);
          break;
        }
        mbar_arrive_expect_tx(&y_full[yb], L::kYPer * L::kYBytes);
        uint8_t* yd = y_buf + yb * L::kYPer * L::kYBytes;
        bulk_load(yd, a.Y0 + yrow * DP * DP, L::kYBytes, &y_full[yb], pol_frame);
        if (L::kYPer == 2)
          bulk_load(yd + L::kYBytes, a.Y1 + yrow * DP * DP, L::kYBytes, &y_full[yb], pol_frame);
        y_fills.filled(yb, yph);
        for (int tile = 0; tile < n_tiles; ++tile) {
          if (!mbar_wait(&empty[stage], phase ^ 1)) {
            give_up(none, abort_flag);
            break;
          }
          mbar_arrive_expect_tx(&full[stage], L::kStageBytes);
          uint8_t* xd = x_ring + stage * L::kStageBytes;
#pragma unroll
          for (int kb = 0; kb < L::kBoxes; ++kb) {
            tma_load_4d(xd + kb * kBoxBytes, &tm_x0, &full[stage], kb * 64, h,
                        tile * kRowsPerTile, bt, pol_stream);
            if (kTerms == 2)
              tma_load_4d(xd + L::kXBytes + kb * kBoxBytes, &tm_x1, &full[stage], kb * 64, h,
                          tile * kRowsPerTile, bt, pol_stream);
          }
          fills.filled(stage, phase);
          if (++stage == L::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      fills.drain(full);
      y_fills.drain(y_full);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc0 = idesc_bf16(128, DP, false, kMN0);
    constexpr uint32_t idesc1 = idesc_bf16(128, DP, false, kMN1);
    int stage = 0;
    uint32_t phase = 0;
    int tc = 0;
    bool ok = true;
    int li = 0;
    for (long item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++li) {
      const int yb = li % L::kYBufs;
      if (!mbar_wait(&y_full[yb], (li / L::kYBufs) & 1)) {
        ok = false;
        break;
      }
      const uint32_t y_base = smem_u32(y_buf + yb * L::kYPer * L::kYBytes);
      // kDualE: this item's E accumulator is free once the epilogue has read item li - 2's
      const uint32_t e_acc = tmem_base + 2 * DP + (li & 1) * DP;
      if (kDualE && !mbar_wait(&e_empty[li & 1], ((li >> 1) & 1) ^ 1)) {
        ok = false;
        break;
      }
      for (int tile = 0; tile < n_tiles; ++tile, ++tc) {
        const int acc = tc & 1;
        if (!mbar_wait(&acc_empty[acc], ((tc >> 1) & 1) ^ 1) || !mbar_wait(&full[stage], phase)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const uint32_t x_base = smem_u32(x_ring + stage * L::kStageBytes);
#pragma unroll
          for (int term = 0; term < kMmaTerms; ++term) {
            const bool mn = term == 0 ? kMN0 : kMN1;
            const uint32_t xb = x_base + term * L::kXBytes;
            const uint32_t yt = y_base + term * L::kYBytes;
#pragma unroll
            for (int ks = 0; ks < DP / 16; ++ks) {
              const uint64_t da = smem_desc(xb + (ks >> 2) * kBoxBytes + (ks & 3) * 32, 16, 1024);
              // s8 frame matrix: K-major (contraction over its keys: key groups 2ks, 2ks+1,
              // DP*16 bytes apart) or MN-major (contraction over its rows: 8-row groups 2ks,
              // 2ks+1, 128 bytes apart; key groups DP*16 bytes apart)
              const uint64_t db = mn ? smem_desc_noswz(yt + ks * 256, 128, DP * 16)
                                     : smem_desc_noswz(yt + ks * 2 * DP * 16, DP * 16, 128);
              mma_bf16(tmem_base + acc * kAccs * DP, da, db, term == 0 ? idesc0 : idesc1,
                       (term | ks) != 0);
            }
          }
          if constexpr (kDualV) {
            // second accumulator: X1 Y0^T, Y0 read K-major
            constexpr uint32_t idesc_k = idesc_bf16(128, DP, false, false);
            const uint32_t xb = x_base + L::kXBytes;
#pragma unroll
            for (int ks = 0; ks < DP / 16; ++ks) {
              const uint64_t da = smem_desc(xb + (ks >> 2) * kBoxBytes + (ks & 3) * 32, 16, 1024);
              const uint64_t db = smem_desc_noswz(y_base + ks * 2 * DP * 16, DP * 16, 128);
              mma_bf16(tmem_base + (acc * kAccs + 1) * DP, da, db, idesc_k, ks != 0);
            }
          }
          if constexpr (kDualE) {
            // E_t += dO^T Q over this tile's 128 tokens: both tiles MN-major (64-dim boxes
            // kBoxBytes apart along M / N, 8-token groups 1024 bytes apart along K)
            constexpr uint32_t idesc_e = idesc_bf16(128, DP, true, true);
#pragma unroll
            for (int ks = 0; ks < kRowsPerTile / 16; ++ks) {
              const uint32_t koff = ks * 16 * 128;  // 16 token rows of 128 B
              const uint64_t da = smem_desc(x_base + koff, kBoxBytes, 1024);
              const uint64_t db = smem_desc(x_base + L::kXBytes + koff, kBoxBytes, 1024);
              mma_bf16(e_acc, da, db, idesc_e, (tile | ks) != 0);
            }
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
      if (elect_one()) {
        if (kDualE) mma_commit(&e_full[li & 1]);
        mma_commit(&y_empty[yb]);
      }
      __syncwarp();
    }
    if (!ok) give_up(none, abort_flag);
    if (elect_one()) mma_commit(mma_drain);
    __syncwarp();
    mbar_wait(mma_drain, 0);
  } else {
    // ---------------------------------------------------------------- epilogue
    const uint32_t quarter = warp & 3;
    const int c0 = ((warp - 2) >> 2) * L::kCols;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem_base + ((quarter * 32) << 16);
    const bool leader = (threadIdx.x == 64);
    const uint64_t pol_out = policy_evict_first();
    if (leader) {
      tma_prefetch_desc(&tm_o);
      if (kDualV) tma_prefetch_desc(&tm_o2);
    }
    int tc = 0;
    int nst = 0;  // staging tiles used (ring position)
    bool ok = true;
    int li = 0;
    for (long item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++li) {
      int bt, h;
      long yrow;
      decode(item, bt, h, yrow);
      const float scale =
          a.beta ? p.key_scale * __ldg(a.beta + static_cast<long>(bt) * p.H + h) : 1.f;
      for (int tile = 0; tile < n_tiles; ++tile, ++tc) {
        const int acc = tc & 1;
        const int valid = min(kRowsPerTile, p.N - tile * kRowsPerTile);
        const bool waited = mbar_wait(&acc_full[acc], (tc >> 1) & 1);
        bool lost = false;
#pragma unroll
        for (int o = 0; o < kAccs; ++o, ++nst) {
          // the staging tile is free once the store issued kOBufs tiles ago has read it
          if (leader) bulk_wait_read<L::kOBufs - 1>();
          if (named_bar_any(1, kEpiThreads, !waited)) {
            lost = true;
            break;
          }
          tc_fence_after();
          uint8_t* ob = o_stage + (nst % L::kOBufs) * L::kOBytes;
          if (static_cast<int>(quarter) * 32 < valid) {
            const uint32_t tacc = lane_base + (acc * kAccs + o) * DP;
            float v[32];
            tmem_ld32(tacc + c0, v);
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              uint4 pk;
              pk.x = pack_bf16x2(v[j] * scale, v[j + 1] * scale);
              pk.y = pack_bf16x2(v[j + 2] * scale, v[j + 3] * scale);
              pk.z = pack_bf16x2(v[j + 4] * scale, v[j + 5] * scale);
              pk.w = pack_bf16x2(v[j + 6] * scale, v[j + 7] * scale);
              *reinterpret_cast<uint4*>(ob + swz128_offset_bf16(row, c0 + j, kBoxBytes)) = pk;
            }
          }
          if (o == kAccs - 1) {
            tc_fence_before();
            mbar_arrive(&acc_empty[acc]);
          }
          fence_async_smem();
          named_bar(1, kEpiThreads);
          if (leader) {
            const CUtensorMap* tmo = o == 0 ? &tm_o : &tm_o2;
#pragma unroll
            for (int kb = 0; kb < L::kBoxes; ++kb)
              tma_store_4d(tmo, ob + kb * kBoxBytes, kb * 64, h, tile * kRowsPerTile, bt,
                           pol_out);
            bulk_commit();
          }
        }
        if (lost) {
          ok = false;
          break;
        }
      }
      if constexpr (kDualE) {
        // E_t of this item: thread = row v of E (TMEM lane), 32 key columns from c0
        if (!ok) break;
        const bool waited = mbar_wait(&e_full[li & 1], (li >> 1) & 1);
        if (named_bar_any(1, kEpiThreads, !waited)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float v[32];
        tmem_ld32(lane_base + 2 * DP + (li & 1) * DP + c0, v);
        tc_fence_before();
        mbar_arrive(&e_empty[li & 1]);
        const int D = p.D;
        if (row < D) {
          float* em = a.E + yrow * D * D;
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            if (c0 + j < D)
              *reinterpret_cast<float4*>(em + b4_index(row, c0 + j, D)) =
                  make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
        }
      }
    }
    if (leader) bulk_wait_all();
    if (!ok) give_up(none, abort_flag);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

}  // namespace gdn
