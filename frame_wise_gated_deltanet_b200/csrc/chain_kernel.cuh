// State chain: S_t = gamma_t * (S_{t-1} - beta_t * S_{t-1} A_t) + beta_t * B_t, frame after
// frame, one CTA per (batch, head). This is the only serial dependency of the layer, so the
// kernel is built for per-frame latency:
//
//   * The identity part of the frame map is kept implicit and exact: S lives in fp32 registers
//     of 16 epilogue warps (thread = one row v of S, a quarter of its columns); only the small
//     correction S_{t-1} A_t goes through the tensor core (S as a bf16 K-major operand written
//     by the epilogue into shared memory, A_t as a bf16 K-major operand loaded by TMA, f32
//     accumulate in TMEM).
//   * B_t is stored in the four-key interleaved layout of b4_index, so each epilogue warp copies
//     its 32 rows x 4 keys as 512 contiguous bytes; every thread copies its own slice with
//     cp.async into one of two shared-memory buffers two frames ahead, and reads it back
//     conflict-free in the same layout.
//   * The bf16 operand tile of S is kept in the no-swizzle core-matrix layout of s8_offset_bytes,
//     which is also the global layout of S_t for the output GEMM: right after handing the tile
//     to the MMA, each thread writes its 16-byte pieces of S_t to global memory (a warp writes
//     512 contiguous bytes per key group), so nothing waits on a store of the tile.
//   * The producer warp checks each frame's hand-off conditions right before loading its A_t and
//     opens that frame's gate (a ring of 8 mbarriers) for the epilogue's B_t copy, so every wait
//     of the chain is on a frame it actually needs next.
//
// Warps: 0..15 epilogue (warp w: rows 32*(w%4).., columns (w/4)*DP/4..), 16 TMA producer and
// gate, 17 TMEM allocator + MMA issuer, 18 publisher (fused only).
//
// Standalone (gdn_chain_kernel): A_t, B_t, S_t at workspace row (b*H+h)*T + t; A_t, B_t of
// later frames are prefetched into L2. The standalone kernel also runs the two per-chunk jobs of
// the chunked forward (ChainSeg): the replay of one chunk of frames from its chunk-start state,
// and the composition of one chunk's affine frame maps (the same recurrence started from the
// identity without B_t, or from zero with B_t). Fused (chain role of gdn_fused_kernel, CTA
// base + b*H + h): rows (b*H+h)*R + t%R of the A/B rings and (b*H+h)*Rs + t%Rs of the S ring;
// frame t is gated on stats_flag (A_t, B_t written) and on out_flag of frame t-Rs (its S slot
// free), and chain_prog is advanced once every thread's part of S_t is visible.
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace gdn {

// What one CTA of the standalone chain kernel computes.
//   kind 0 (replay): frames [c*L, min(T, (c+1)*L)) of head bh = blockIdx.x / nc, chunk
//     c = blockIdx.x % nc, starting from state_in (nc == 1) or from the chunk-start state of
//     record bh*nc + c in `starts` (layout at chunk_start_bytes, written by the inter-chunk
//     scan; record 0 is the scan's copy of state_in); writes S_t of every frame and, for the
//     clip's last chunk, state_out.
//     With L = T and nc = 1 this is the plain per-head chain.
//   kind 1 (composition): chunk c < nc - 1 of head bh, CTA pair (2*(bh*(nc-1) + c) + role).
//     Frame t maps a state to S * M_t + C_t with M_t = gamma_t (I - beta_t A_t) and
//     C_t = beta_t B_t; the same recurrence started from the identity without B_t yields
//     P_c = M_{cL} ... M_{cL+L-1} (role 0), started from zero with B_t it yields the offset C_c
//     (role 1), so the chunk's end state is S_start * P_c + C_c. Both go to the chunk's record
//     in `maps` (layout at chunk_map_bytes).
struct ChainSeg {
  int L;
  int nc;
  int kind;
  uint8_t* maps;
  uint8_t* starts;
};

template <int DP>
struct ChainLayout {
  static constexpr int kABytes = DP * DP * 2;   // A_t bf16: DP/64 blocks of DP rows x 128 B
  static constexpr int kStages = 2;             // A_t stages
  static constexpr int kBBufBytes = DP * 512;   // B_t f32: [DP/4 key groups][128 rows][16 B]
  static constexpr int kBBufs = 2;
  static constexpr int kGate = 8;               // gate ring
  static constexpr int kSBytes = DP * 256;      // S operand: [DP/8 key groups][128 rows][16 B]
  static constexpr int kEpiWarps = 16;
  static constexpr int kThreads = (kEpiWarps + 3) * 32;
  static constexpr int kWarpProducer = kEpiWarps;
  static constexpr int kWarpMma = kEpiWarps + 1;
  static constexpr int kWarpPublisher = kEpiWarps + 2;
  static constexpr int kCols = DP / 4;  // columns of S per epilogue thread
  static constexpr int kTmemCols = 128;
  static constexpr int kSmemBytes = kStages * kABytes + kBBufs * kBBufBytes + kSBytes + 512 + 1024;
};

// S_out: bf16 states, one DP*DP block per row (workspace or ring), layout of s8_offset_bytes.
template <int DP, bool kFused>
__device__ __forceinline__ void chain_body(const CUtensorMap* tm_a, const float* __restrict__ B_ws,
                                           __nv_bfloat16* __restrict__ S_out,
                                           const float* __restrict__ gamma,
                                           const float* __restrict__ beta,
                                           const float* __restrict__ state_in,
                                           float* __restrict__ state_out, const Problem& p,
                                           const Handoff& hf, const ChainSeg& seg,
                                           uint8_t* smem) {
  using L = ChainLayout<DP>;
  uint8_t* b_buf = smem + L::kStages * L::kABytes;
  uint8_t* s_tile = b_buf + L::kBBufs * L::kBBufBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(s_tile + L::kSBytes);
  uint64_t* empty = full + L::kStages;
  uint64_t* gate = empty + L::kStages;   // frame f (slot f % kGate) may be read and written
  uint64_t* mma_done = gate + L::kGate;
  uint64_t* s_ready = mma_done + 1;      // the S tile holds the new state
  // fused: epilogue warps that have written their part of S_t to global memory, summed over
  // frames (kEpiWarps per frame); a counter, not a barrier, so the publisher may lag freely
  uint64_t* mma_drain = s_ready + 1;     // all of this CTA's MMAs are complete
  uint32_t* s_written = reinterpret_cast<uint32_t*>(mma_drain + 1);
  uint32_t* tmem_slot = s_written + 1;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int T = p.T;
  const int D = p.D;
  const long DD = static_cast<long>(D) * D;
  // this CTA's head, chunk and frames [t0, t1); the pointers it reads and writes are derived
  // at their point of use (chunk_state) so that nothing extra stays live across the frame loop
  int bh, chunk = 0, t0 = 0, t1 = T, map_role = -1;
  if (kFused) {
    bh = static_cast<int>(blockIdx.x) - hf.base;
  } else if (seg.kind == 0) {
    bh = static_cast<int>(blockIdx.x) / seg.nc;
    chunk = static_cast<int>(blockIdx.x) - bh * seg.nc;
    t0 = chunk * seg.L;
    t1 = min(T, t0 + seg.L);
  } else {
    const int item = static_cast<int>(blockIdx.x) >> 1;
    map_role = static_cast<int>(blockIdx.x) & 1;
    bh = item / (seg.nc - 1);
    chunk = item - bh * (seg.nc - 1);
    t0 = chunk * seg.L;
    t1 = t0 + seg.L;
  }
  const bool identity = map_role == 0;  // composition of P_c: start from I, no B_t
  const bool use_b = map_role != 0;
  // start state (nullptr: zero) and final state (nullptr: not stored) of this CTA
  // start state from the scan's records (chunked replay) instead of state_in
  const bool start_from_record = !kFused && map_role < 0 && seg.nc > 1;
  auto init_state = [&]() -> const float* {  // row-major f32 start state, nullptr: zero
    if (map_role >= 0 || start_from_record) return nullptr;
    return state_in ? state_in + bh * DD : nullptr;
  };
  auto final_state = [&]() -> float* {
    if (kFused || (map_role < 0 && chunk == seg.nc - 1)) return state_out ? state_out + bh * DD : nullptr;
    return nullptr;
  };
  const int n = t1 - t0;  // frames of this CTA; loop counters below are local (0..n-1)
  const bool write_s = S_out != nullptr;
  const int b = bh / p.H;
  const int h = bh - b * p.H;
  // row of frame f's A_t / B_t, and of its S_t
  auto row_of = [&](int f) { return kFused ? bh * hf.R + f % hf.R : bh * T + f; };
  auto srow_of = [&](int f) { return kFused ? bh * hf.Rs + f % hf.Rs : bh * T + f; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < L::kGate; ++s) mbar_init(&gate[s], 1);
    mbar_init(mma_done, 1);
    mbar_init(s_ready, L::kEpiWarps);  // one arrival per epilogue warp
    mbar_init(mma_drain, 1);
    *s_written = 0;
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
    // ---------------------------------------------------------------- gate, A_t via TMA
    if (elect_one()) {
      tma_prefetch_desc(tm_a);
      const uint64_t pol = kFused ? policy_evict_last() : policy_evict_first();
      constexpr int kPrefetch = 8;  // standalone: frames pulled into L2 ahead of use
      auto prefetch = [&](int f) {  // f: frame index
#pragma unroll
        for (int kb = 0; kb < DP / 64; ++kb) tma_prefetch_3d(tm_a, kb * 64, 0, row_of(f));
        if (use_b)
          bulk_prefetch_l2(B_ws + static_cast<long>(row_of(f)) * D * D,
                           static_cast<uint32_t>(D * D * 4));
      };
      if constexpr (!kFused)
        for (int u = 0; u < kPrefetch && u < n; ++u) prefetch(t0 + u);
      // Gate frame t, then load A_t. Fused: frame t's A_t, B_t must be published and the output
      // of frame t-Rs must have loaded S_{t-Rs} from the slot S_t will use. Gate slot
      // t % kGate was last used by frame t - kGate, whose B copy the epilogue issued at step
      // t - kGate - 2, before the MMA of step t - 2 that the empty-stage wait below follows.
      StageFills<L::kStages> fills;
      for (int u = 0; u < n; ++u) {
        const int t = t0 + u;
        const int stage = u % L::kStages;
        const uint32_t phase = (u / L::kStages) & 1;
        if constexpr (!kFused) {
          if (u + kPrefetch < n) prefetch(t + kPrefetch);
        }
        bool ok = mbar_wait(&empty[stage], phase ^ 1);
        if constexpr (kFused) {
          ok = ok && wait_flag_ge(hf.stats_flag + static_cast<long>(bh) * T + t, 1, hf.abort);
          ok = ok && (t < hf.Rs || wait_flag_ge(hf.out_flag + static_cast<long>(bh) * T + t - hf.Rs,
                                                1, hf.abort));
          fence_async_global();
        }
        if (!ok) {
          give_up(hf, abort_flag);
          break;
        }
        mbar_arrive(&gate[u % L::kGate]);
        mbar_arrive_expect_tx(&full[stage], L::kABytes);
        uint8_t* st = smem + stage * L::kABytes;
        const int row = row_of(t);
#pragma unroll
        for (int kb = 0; kb < DP / 64; ++kb)
          tma_load_3d(st + kb * DP * 128, tm_a, &full[stage], kb * 64, 0, row, pol);
        fills.filled(stage, phase);
      }
      fills.drain(full);  // this thread's copies have landed, whatever the exit path
    }
  } else if (warp == L::kWarpMma) {
    // ---------------------------------------------------------------- MMA: P = S_{t-1} A_t
    constexpr uint32_t idesc = idesc_bf16(128, DP, false, false);
    // Operand descriptors built once (the step's issue is on the chain's path); a k-step adds its
    // byte offset / 16 to the start-address field, which stays below 2^14 inside shared memory.
    // S tile: key groups 2ks, 2ks+1 (2048 B apart), 8-row groups 128 B apart.
    // A_t stages: 128B-swizzled, 64-key blocks of DP rows.
    const uint64_t da0 = smem_desc_noswz(smem_u32(s_tile), 2048, 128);
    const uint64_t db0 = smem_desc(smem_u32(smem), 16, 1024);
    static_assert(L::kStages == 2, "stage descriptors");
    bool ok = true;
    for (int u = 0; u < n; ++u) {
      const int stage = u % L::kStages;
      const uint32_t phase = (u / L::kStages) & 1;
      if (!mbar_wait(&full[stage], phase) || !mbar_wait(s_ready, u & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (elect_one()) {
        const uint64_t dbs = db0 + (stage ? (L::kABytes >> 4) : 0);
#pragma unroll
        for (int ks = 0; ks < DP / 16; ++ks)
          mma_bf16(tmem_base, da0 + ((ks * 2 * 2048) >> 4),
                   dbs + (((ks >> 2) * DP * 128 + (ks & 3) * 32) >> 4), idesc, ks != 0);
        mma_commit(mma_done);
        mma_commit(&empty[stage]);
      }
      __syncwarp();
    }
    if (!ok) give_up(hf, abort_flag);
    // every MMA issued here has completed before TMEM is released
    if (elect_one()) mma_commit(mma_drain);
    __syncwarp();
    mbar_wait(mma_drain, 0);
  } else if (warp == L::kWarpPublisher) {
    // ---------------------------------------------------------------- fused: publish S_t
    if constexpr (kFused) {
      if (elect_one()) {
        int published = 0;
        unsigned long long t0 = globaltimer_ns();
        // queue position of the next frame, reserved a frame ahead so that publishing costs no
        // atomic round trip (positions still follow the order in which frames are published)
        int pos = atomicAdd(hf.ready_tail, 1);
        while (published < T) {
          const int done = static_cast<int>(ld_acquire_cta(s_written) / L::kEpiWarps);
          if (done > published) {
            // every epilogue warp's S stores happen-before its release-add, which this thread
            // has acquired; the GPU-scope release makes them visible to the outputs (which
            // fence the async proxy after their acquire)
            st_release(hf.chain_prog + bh, done);
            // queue the frames for the outputs: a plain store suffices, since an output acquires
            // chain_prog itself before it reads S_t
            for (int f = published; f < done; ++f) {
              st_relaxed(hf.ready_items + pos, f * p.B * p.H + bh + 1);
              if (f + 1 < T) pos = atomicAdd(hf.ready_tail, 1);
            }
            published = done;
            t0 = globaltimer_ns();
            continue;
          }
          if (*abort_flag || ld_acquire(hf.abort) != 0 || globaltimer_ns() - t0 > g_wait_limit_ns) {
            give_up(hf, abort_flag);
            break;
          }
          __nanosleep(32);
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue (512 threads)
    const uint32_t quarter = warp & 3;
    const int v = quarter * 32 + lane;              // row of S (value index)
    const int c0 = (warp >> 2) * L::kCols;          // first column (key index) owned
    const uint32_t taddr = tmem_base + ((quarter * 32) << 16) + c0;
    const bool row_ok = v < D;
    float S[L::kCols];
    if (start_from_record) {
      // chunk-start state from the scan, four-key interleaved (coalesced 16-byte reads)
      const float* rec = reinterpret_cast<const float*>(
          seg.starts + (static_cast<long>(bh) * seg.nc + chunk) * chunk_start_bytes(DP));
#pragma unroll
      for (int j = 0; j < L::kCols; j += 4) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (row_ok && c0 + j < D) x = __ldcg(reinterpret_cast<const float4*>(rec + b4_index(v, c0 + j, D)));
        S[j] = x.x;
        S[j + 1] = x.y;
        S[j + 2] = x.z;
        S[j + 3] = x.w;
      }
    } else {
      const float* s0 = init_state();
      const float* sin = s0 ? s0 + static_cast<long>(v) * D : nullptr;
#pragma unroll
      for (int j = 0; j < L::kCols; ++j) {
        const int col = c0 + j;
        const bool in = row_ok && col < D;
        S[j] = identity ? (in && col == v ? 1.f : 0.f) : ((sin != nullptr && in) ? sin[col] : 0.f);
      }
    }
    auto pack8 = [&](int j) {
      uint4 pk;
      pk.x = pack_bf16x2(S[j], S[j + 1]);
      pk.y = pack_bf16x2(S[j + 2], S[j + 3]);
      pk.z = pack_bf16x2(S[j + 4], S[j + 5]);
      pk.w = pack_bf16x2(S[j + 6], S[j + 7]);
      return pk;
    };
    auto write_s_tile = [&]() {
#pragma unroll
      for (int j = 0; j < L::kCols; j += 8)
        *reinterpret_cast<uint4*>(s_tile + ((c0 + j) >> 3) * 2048 + v * 16) = pack8(j);
    };
    // this thread's 16-byte group kg of row v in a B buffer
    auto b_slot = [&](int buf, int kg) {
      return b_buf + buf * L::kBBufBytes + (static_cast<uint32_t>(kg) * 128 + v) * 16;
    };
    // copy this thread's slice of B of local frame f (from L2) into buffer f % 2, one commit
    // group per frame
    auto issue_b = [&](int f) -> bool {
      if (!mbar_wait(&gate[f % L::kGate], (f / L::kGate) & 1)) return false;
      const float* bm = B_ws + static_cast<long>(row_of(t0 + f)) * D * D;
      if (row_ok && use_b) {
#pragma unroll
        for (int j = 0; j < L::kCols; j += 4) {
          const int col = c0 + j;
          if (col < D) cp_async16(b_slot(f & 1, col >> 2), bm + b4_index(v, col, D));
        }
      }
      cp_async_commit();
      return true;
    };
    write_s_tile();
    fence_async_smem();
    tc_fence_before();
    bool ok = issue_b(0);
    if (ok) {
      if (n > 1)
        ok = issue_b(1);
      else
        cp_async_commit();
    }
    __syncwarp();  // the warp's tile writes and fences first
    if (lane == 0) mbar_arrive(s_ready);

    // gamma_t, beta_t: each lane holds frame (32*blk + lane) of the current and next block of
    // 32 frames; the value for frame t is shuffled from lane t % 32.
    const long gb_base = static_cast<long>(b) * T * p.H + h;
    auto load_gb = [&](int blk, float& gv, float& bv) {
      const int f = t0 + blk * 32 + static_cast<int>(lane);
      gv = f < t1 ? __ldg(gamma + gb_base + static_cast<long>(f) * p.H) : 0.f;
      bv = f < t1 ? __ldg(beta + gb_base + static_cast<long>(f) * p.H) : 0.f;
    };
    float g_cur, b_cur, g_next, b_next;
    load_gb(0, g_next, b_next);
    for (int u = 0; u < n && ok; ++u) {
      const int t = t0 + u;
      if ((u & 31) == 0) {
        g_cur = g_next;
        b_cur = b_next;
        load_gb((u >> 5) + 1, g_next, b_next);
      }
      const float g = __shfl_sync(0xffffffffu, g_cur, u & 31);
      const float be = __shfl_sync(0xffffffffu, b_cur, u & 31);
      // S_t = gamma_t S_{t-1} + beta_t B_t - gamma_t beta_t S_{t-1} A_t: the part that does not
      // need the product is formed while the MMA runs, so that one FMA per element follows the
      // wait (the step is the chain's latency)
      cp_async_wait<1>();  // this thread's copy of B_t (B_{t+1} may still be in flight)
#pragma unroll
      for (int j = 0; j < L::kCols; j += 4) {
        float4 bv = make_float4(0.f, 0.f, 0.f, 0.f);
        if (use_b && row_ok && c0 + j < D)
          bv = *reinterpret_cast<const float4*>(b_slot(u & 1, (c0 + j) >> 2));
        S[j] = fmaf(g, S[j], be * bv.x);
        S[j + 1] = fmaf(g, S[j + 1], be * bv.y);
        S[j + 2] = fmaf(g, S[j + 2], be * bv.z);
        S[j + 3] = fmaf(g, S[j + 3], be * bv.w);
        // at most 16 columns of B_t in registers at a time (the reads of the next 16 may not
        // be hoisted above this point), which the fused kernel's register budget needs
        if ((j & 15) == 12) asm volatile("" ::: "memory");
      }
      if (!mbar_wait(mma_done, u & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float ngbe = -g * be;
#pragma unroll
      for (int c = 0; c < L::kCols; c += 16) {
        float P[16];
        tmem_ld16(taddr + c, P);
#pragma unroll
        for (int j = 0; j < 16; ++j) S[c + j] = fmaf(ngbe, P[j], S[c + j]);
      }
      write_s_tile();
      fence_async_smem();
      tc_fence_before();
      __syncwarp();  // the warp's tile writes and fences first
      if (lane == 0) mbar_arrive(s_ready);
      // S_t to global (its slot was gated free): rows past D and M-padding rows hold zeros,
      // rows >= DP (M-padding when DP == 64) are not part of the stored matrix
      if (write_s && v < DP) {
        uint8_t* srow = reinterpret_cast<uint8_t*>(S_out + static_cast<long>(srow_of(t)) * DP * DP);
#pragma unroll
        for (int j = 0; j < L::kCols; j += 8)
          *reinterpret_cast<uint4*>(srow + s8_offset_bytes(v, c0 + j, DP)) = pack8(j);
      }
      if constexpr (kFused) {
        __syncwarp();  // the warp's S stores before its lane 0's release-add
        if (lane == 0) red_add_release_cta(s_written, 1);
      }
      // buffer u % 2 is free (this thread read its own slice above): copy B of frame u + 2
      if (u + 2 < n) {
        if (!issue_b(u + 2)) {
          ok = false;
          break;
        }
      } else {
        cp_async_commit();
      }
    }
    cp_async_wait<0>();
    if (!ok) give_up(hf, abort_flag);
    float* const s_end = final_state();
    if (ok && s_end != nullptr && row_ok) {
      float* so = s_end + static_cast<long>(v) * D;
#pragma unroll
      for (int j = 0; j < L::kCols; j += 4)
        if (c0 + j < D)
          *reinterpret_cast<float4*>(so + c0 + j) = make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
    }
    uint8_t* const map_dst = map_role >= 0 ? seg.maps + (static_cast<long>(bh) * (seg.nc - 1) + chunk) *
                                                         chunk_map_bytes(DP)
                                           : nullptr;
    if (ok && map_role == 0 && v < DP) {
      // P_c transposed, split into bf16 hi + lo, as the scan's K-major B operand: element
      // (n, k) = P_c[k][n] at s8_offset_bytes(n, k); this thread holds P_c row k = v
#pragma unroll
      for (int j = 0; j < L::kCols; ++j) {
        const __nv_bfloat16 hi = __float2bfloat16_rn(S[j]);
        const __nv_bfloat16 lo = __float2bfloat16_rn(S[j] - __bfloat162float(hi));
        const long off = s8_offset_bytes(c0 + j, v, DP);
        *reinterpret_cast<__nv_bfloat16*>(map_dst + off) = hi;
        *reinterpret_cast<__nv_bfloat16*>(map_dst + DP * DP * 2 + off) = lo;
      }
    }
    if (ok && map_role == 1 && row_ok) {
      // C_c in the four-key interleaved layout of b4_index (read back like B_t)
      float* cm = reinterpret_cast<float*>(map_dst + 2 * DP * DP * 2);
#pragma unroll
      for (int j = 0; j < L::kCols; j += 4)
        if (c0 + j < D)
          *reinterpret_cast<float4*>(cm + b4_index(v, c0 + j, D)) =
              make_float4(S[j], S[j + 1], S[j + 2], S[j + 3]);
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
                     __nv_bfloat16* __restrict__ S_ws, const float* __restrict__ gamma,
                     const float* __restrict__ beta, const float* __restrict__ state_in,
                     float* __restrict__ state_out, Problem p, ChainSeg seg) {
  extern __shared__ uint8_t smem_raw[];
  const Handoff none{nullptr, nullptr, nullptr, nullptr, nullptr, 1, 1, -1, 0, 0};
  chain_body<DP, false>(&tm_a, B_ws, S_ws, gamma, beta, state_in, state_out, p, none, seg,
                        align1k(smem_raw));
}

}  // namespace gdn
