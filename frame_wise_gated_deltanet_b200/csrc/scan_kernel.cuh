// Inter-chunk scan of the chunked forward. Chunk c of head bh maps its start state to its end
// state as S_end = S_start * P_c + C_c (P_c, C_c: the composed affine frame maps of the chunk,
// written by the composition CTAs of gdn_chain_kernel). This kernel walks the chunks of one head
// in order, one CTA per (batch, head), and writes the start state of every chunk c >= 1 for the
// per-chunk replay. Only ceil(T / L) - 1 dependent steps remain on the serial path instead of T.
//
// Precision: unlike the frame maps, P_c is not close to the identity times a small correction
// (its diagonal is the product of the chunk's gammas), so S * P_c is computed from bf16 hi/lo
// splits of both factors, S_hi P_hi + S_hi P_lo + S_lo P_hi, accumulated in f32 in TMEM. The
// dropped S_lo P_lo term is about 2^-16 of the product. S itself stays f32 in registers.
//
// The epilogue stores every chunk-start state in the four-key interleaved layout (512 contiguous
// bytes per warp and store). Row-major stores (128 bytes per lane, lanes a row apart) doubled
// the step time, and a bulk copy of the shared-memory operand tiles by the MMA thread was slower
// than these coalesced stores.
//
// Warps: 0..15 epilogue (thread = row v of S, DP/4 columns), 16 bulk-copy producer of the P_c
// records (two stages), 17 TMEM allocator + MMA issuer.
#pragma once
#include "common.cuh"

namespace gdn {

template <int DP>
struct ScanLayout {
  static constexpr int kPBytes = 2 * DP * DP * 2;  // P_c hi + lo (bf16, s8 layout)
  static constexpr int kStages = 2;
  static constexpr int kSBytes = DP * 256;         // one S operand tile: [DP/8][128 rows][16 B]
  static constexpr int kEpiWarps = 16;
  static constexpr int kThreads = (kEpiWarps + 2) * 32;
  static constexpr int kWarpProducer = kEpiWarps;
  static constexpr int kWarpMma = kEpiWarps + 1;
  static constexpr int kCols = DP / 4;
  static constexpr int kTmemCols = 128;
  static constexpr int kSmemBytes = kStages * kPBytes + 2 * kSBytes + 256 + 1024;
};

// maps: nc - 1 records per head (chunk_map_bytes(DP) each); starts: nc records per head
// (chunk_start_bytes(DP) each); record bh*nc + c receives the start state of chunk c (record 0:
// a copy of state_in, so that the replays never read state_in while the last one writes
// state_out, which may be the same memory).
template <int DP>
__global__ void __launch_bounds__(ScanLayout<DP>::kThreads, 1)
    gdn_scan_kernel(const uint8_t* __restrict__ maps, uint8_t* __restrict__ starts,
                    const float* __restrict__ state_in, int nc, int D) {
  using L = ScanLayout<DP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1k(smem_raw);
  uint8_t* s_hi = smem + L::kStages * L::kPBytes;
  uint8_t* s_lo = s_hi + L::kSBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(s_lo + L::kSBytes);
  uint64_t* empty = full + L::kStages;
  uint64_t* mma_done = empty + L::kStages;
  uint64_t* s_ready = mma_done + 1;
  uint64_t* mma_drain = s_ready + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int bh = blockIdx.x;
  const int steps = nc - 1;
  const long DD = static_cast<long>(D) * D;
  const uint8_t* head_maps = maps + static_cast<long>(bh) * steps * chunk_map_bytes(DP);
  const Handoff none{nullptr, nullptr, nullptr, nullptr, nullptr, 1, 1, -1, 0, 0};

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(mma_done, 1);
    mbar_init(s_ready, L::kEpiWarps);  // one arrival per epilogue warp
    mbar_init(mma_drain, 1);
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
    // ---------------------------------------------------------------- P_c records, bulk copies
    if (elect_one()) {
      const uint64_t pol = policy_evict_first();
      StageFills<L::kStages> fills;
      for (int c = 0; c < steps; ++c) {
        const int stage = c % L::kStages;
        const uint32_t phase = (c / L::kStages) & 1;
        if (!mbar_wait(&empty[stage], phase ^ 1)) {
          give_up(none, abort_flag);
          break;
        }
        const uint8_t* rec = head_maps + static_cast<long>(c) * chunk_map_bytes(DP);
        mbar_arrive_expect_tx(&full[stage], L::kPBytes);
        bulk_load(smem + stage * L::kPBytes, rec, L::kPBytes, &full[stage], pol);
        fills.filled(stage, phase);
        // the C_c part of the next records, read by the epilogue straight from L2
        if (c + 2 < steps)
          bulk_prefetch_l2(rec + 2 * chunk_map_bytes(DP) + L::kPBytes,
                           static_cast<uint32_t>(DP * DP * 4));
      }
      fills.drain(full);
    }
  } else if (warp == L::kWarpMma) {
    // ---------------------------------------------------------------- MMA: S * P_c (3 passes)
    constexpr uint32_t idesc = idesc_bf16(128, DP, false, false);
    bool ok = true;
    for (int c = 0; c < steps; ++c) {
      const int stage = c % L::kStages;
      const uint32_t phase = (c / L::kStages) & 1;
      if (!mbar_wait(&full[stage], phase) || !mbar_wait(s_ready, c & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (elect_one()) {
        const uint32_t p_hi = smem_u32(smem + stage * L::kPBytes);
        const uint32_t p_lo = p_hi + DP * DP * 2;
#pragma unroll
        for (int pass = 0; pass < 3; ++pass) {
          const uint32_t a = pass == 2 ? smem_u32(s_lo) : smem_u32(s_hi);
          const uint32_t bb = pass == 1 ? p_lo : p_hi;
#pragma unroll
          for (int ks = 0; ks < DP / 16; ++ks) {
            // S tile: key groups 2048 B apart; P_c^T: key groups DP*16 B apart
            const uint64_t da = smem_desc_noswz(a + ks * 2 * 2048, 2048, 128);
            const uint64_t db = smem_desc_noswz(bb + ks * 2 * DP * 16, DP * 16, 128);
            mma_bf16(tmem_base, da, db, idesc, (pass | ks) != 0);
          }
        }
        mma_commit(mma_done);
        mma_commit(&empty[stage]);
      }
      __syncwarp();
    }
    if (!ok) give_up(none, abort_flag);
    if (elect_one()) mma_commit(mma_drain);
    __syncwarp();
    mbar_wait(mma_drain, 0);
  } else {
    // ---------------------------------------------------------------- epilogue (512 threads)
    const uint32_t quarter = warp & 3;
    const int v = quarter * 32 + lane;
    const int c0 = (warp >> 2) * L::kCols;
    const uint32_t taddr = tmem_base + ((quarter * 32) << 16) + c0;
    const bool row_ok = v < D;
    float S[L::kCols];
    const float* sin = state_in ? state_in + static_cast<long>(bh) * DD + static_cast<long>(v) * D
                                : nullptr;
#pragma unroll
    for (int j = 0; j < L::kCols; ++j)
      S[j] = (sin != nullptr && row_ok && c0 + j < D) ? sin[c0 + j] : 0.f;
    // start state of chunk 0
    auto store_start = [&](int c) {
      if (!row_ok) return;
      float* so = reinterpret_cast<float*>(
          starts + (static_cast<long>(bh) * nc + c) * chunk_start_bytes(DP));
#pragma unroll
      for (int j = 0; j < L::kCols; j += 4)
        if (c0 + j < D)
          __stcg(reinterpret_cast<float4*>(so + b4_index(v, c0 + j, D)),
                 make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]));
    };
    store_start(0);
    // S as bf16 hi and lo operand tiles (core-matrix layout, rows past D are zero)
    auto write_tiles = [&]() {
#pragma unroll
      for (int j = 0; j < L::kCols; j += 8) {
        float lo[8];
        uint4 h;
        uint32_t* hw = reinterpret_cast<uint32_t*>(&h);
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          const __nv_bfloat16 a = __float2bfloat16_rn(S[j + e]);
          const __nv_bfloat16 b = __float2bfloat16_rn(S[j + e + 1]);
          lo[e] = S[j + e] - __bfloat162float(a);
          lo[e + 1] = S[j + e + 1] - __bfloat162float(b);
          hw[e / 2] = static_cast<uint32_t>(__bfloat16_as_ushort(a)) |
                      (static_cast<uint32_t>(__bfloat16_as_ushort(b)) << 16);
        }
        uint4 l;
        l.x = pack_bf16x2(lo[0], lo[1]);
        l.y = pack_bf16x2(lo[2], lo[3]);
        l.z = pack_bf16x2(lo[4], lo[5]);
        l.w = pack_bf16x2(lo[6], lo[7]);
        const uint32_t off = ((c0 + j) >> 3) * 2048 + v * 16;
        *reinterpret_cast<uint4*>(s_hi + off) = h;
        *reinterpret_cast<uint4*>(s_lo + off) = l;
      }
    };
    bool ok = true;
    if (steps > 0) {
      write_tiles();
      fence_async_smem();
      tc_fence_before();
      __syncwarp();  // the warp's tile writes and fences first
      if (lane == 0) mbar_arrive(s_ready);
    }
    for (int c = 0; c < steps; ++c) {
      // this thread's slice of C_c, loaded while the MMA runs
      const float* cm = reinterpret_cast<const float*>(
          head_maps + static_cast<long>(c) * chunk_map_bytes(DP) + L::kPBytes);
      float C[L::kCols];
#pragma unroll
      for (int j = 0; j < L::kCols; j += 4) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (row_ok && c0 + j < D) x = __ldcg(reinterpret_cast<const float4*>(cm + b4_index(v, c0 + j, D)));
        C[j] = x.x;
        C[j + 1] = x.y;
        C[j + 2] = x.z;
        C[j + 3] = x.w;
      }
      if (!mbar_wait(mma_done, c & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < L::kCols; cc += 16) {
        float P[16];
        tmem_ld16(taddr + cc, P);
#pragma unroll
        for (int j = 0; j < 16; ++j) S[cc + j] = P[j] + C[cc + j];
      }

      if (c + 1 < steps) {
        write_tiles();
        fence_async_smem();
        tc_fence_before();
        __syncwarp();  // the warp's tile writes and fences first
        if (lane == 0) mbar_arrive(s_ready);
      }
      store_start(c + 1);
    }
    if (!ok) give_up(none, abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == L::kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

}  // namespace gdn
