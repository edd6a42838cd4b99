// Backward state chain: the gradient of the loss with respect to every state S_t, walked from
// the last frame to the first, one CTA per (batch, head).
//
// With G_t = dL/dS_t (everything that reaches S_t: the frame's own output O_t = Q_t S_t^T and
// the later frames through S_{t+1} = gamma_{t+1} S_t (I - beta_{t+1} A_{t+1}) + ...):
//
//   G_{T-1} = dS_T + E_{T-1}
//   G_{t-1} = gamma_t * (G_t - beta_t * G_t A_t) + E_{t-1}       (t = T-1 .. 1)
//   dS_0    = gamma_0 * (G_0 - beta_0 * G_0 A_0)
//
// where E_t = dO_t^T Q_t (the output's contribution; the statistics kernel computes it as the
// "B" statistic of (key = q, value = dO) with key scale 1) and A_t = K'^T K' is the forward's
// statistic. It is the forward recurrence run backwards, with the frame map transposed (A_t is
// symmetric, so G (I - beta A)^T = G (I - beta A)) and the additive term E_{t-1} with weight 1.
//
// The design is the forward chain's: G lives in fp32 registers of 16 epilogue warps (thread =
// row v, a quarter of the columns); only the correction G_t A_t goes through the tensor core
// (G as a bf16 operand written by the epilogue into shared memory in the core-matrix layout of
// s8_offset_bytes, A_t by TMA with 128B swizzle, f32 in TMEM); E_{t-1} is copied by every
// thread for its own slice with cp.async (four-key interleaved layout) two frames ahead. Every
// G_t is also written to global memory as bf16 in the s8 layout, for the gradient GEMMs.
//
// A launch may cover a segment of frames [t_lo, t_hi) (walked from t_hi - 1 down to t_lo): it
// starts from dS_T + E_{T-1} when t_hi = T, else from G_{t_hi-1} carried in f32 by the previous
// segment's launch, and it ends with dS_0 when t_lo = 0, else with G_{t_lo-1} carried to the
// next launch. The gradient passes of a finished segment then run while the chain continues.
//
// Warps: 0..15 epilogue, 16 TMA producer of A_t, 17 TMEM allocator + MMA issuer.
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace gdn {

template <int DP>
struct BwdChainLayout {
  static constexpr int kABytes = DP * DP * 2;   // A_t bf16: DP/64 blocks of DP rows x 128 B
  static constexpr int kStages = 2;             // A_t stages
  static constexpr int kEBufBytes = DP * 512;   // E f32: [DP/4 key groups][128 rows][16 B]
  static constexpr int kEBufs = 2;
  static constexpr int kGBytes = DP * 256;      // G operand: [DP/8 key groups][128 rows][16 B]
  static constexpr int kEpiWarps = 16;
  static constexpr int kThreads = (kEpiWarps + 2) * 32;
  static constexpr int kWarpProducer = kEpiWarps;
  static constexpr int kWarpMma = kEpiWarps + 1;
  static constexpr int kCols = DP / 4;
  static constexpr int kTmemCols = 128;
  static constexpr int kSmemBytes = kStages * kABytes + kEBufs * kEBufBytes + kGBytes + 512 + 1024;
};

// A_t: through tm_a, rows (b*H+h)*T + t of the forward statistics; E_ws: f32 D x D per row
// (b4_index layout); G_out: bf16 DP x DP per row (s8 layout); d_state_out / d_state_in: f32
// [B*H][D][D] row-major, nullptr = zero / not stored; carry: f32 [B*H][D][D] row-major, read
// when t_hi < T and written when t_lo > 0 (the same memory is read and then written by the
// same thread, so one buffer serves every segment).
template <int DP>
__global__ void __launch_bounds__(BwdChainLayout<DP>::kThreads, 1)
    gdn_bwd_chain_kernel(const __grid_constant__ CUtensorMap tm_a, const float* __restrict__ E_ws,
                         __nv_bfloat16* __restrict__ G_out, const float* __restrict__ gamma,
                         const float* __restrict__ beta, const float* __restrict__ d_state_out,
                         float* __restrict__ d_state_in, float* carry, int t_lo, int t_hi,
                         Problem p) {
  using L = BwdChainLayout<DP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1k(smem_raw);
  uint8_t* e_buf = smem + L::kStages * L::kABytes;
  uint8_t* g_tile = e_buf + L::kEBufs * L::kEBufBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(g_tile + L::kGBytes);
  uint64_t* empty = full + L::kStages;
  uint64_t* mma_done = empty + L::kStages;
  uint64_t* g_ready = mma_done + 1;   // the G tile holds the next operand
  uint64_t* mma_drain = g_ready + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int T = p.T;
  const int D = p.D;
  const long DD = static_cast<long>(D) * D;
  const int bh = blockIdx.x;
  const int b = bh / p.H;
  const int h = bh - b * p.H;
  const Handoff none{nullptr, nullptr, nullptr, nullptr, nullptr, 1, 1, -1, 0, 0};
  const int n = t_hi - t_lo;  // steps of this launch
  // step u handles frame t = t_hi-1-u: its MMA is G_t A_t
  auto row_of = [&](int t) { return static_cast<long>(bh) * T + t; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(mma_done, 1);
    mbar_init(g_ready, L::kEpiWarps);  // one arrival per epilogue warp
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
    // ---------------------------------------------------------------- A_t via TMA, last first
    if (elect_one()) {
      tma_prefetch_desc(&tm_a);
      const uint64_t pol = policy_evict_first();
      constexpr int kPrefetch = 8;
      auto prefetch = [&](int t) {
#pragma unroll
        for (int kb = 0; kb < DP / 64; ++kb)
          tma_prefetch_3d(&tm_a, kb * 64, 0, static_cast<int>(row_of(t)));
        if (t >= 1)
          bulk_prefetch_l2(E_ws + row_of(t - 1) * DD, static_cast<uint32_t>(DD * 4));
      };
      for (int u = 0; u < kPrefetch && u < n; ++u) prefetch(t_hi - 1 - u);
      StageFills<L::kStages> fills;
      for (int u = 0; u < n; ++u) {
        const int t = t_hi - 1 - u;
        const int stage = u % L::kStages;
        const uint32_t phase = (u / L::kStages) & 1;
        if (u + kPrefetch < n) prefetch(t - kPrefetch);
        if (!mbar_wait(&empty[stage], phase ^ 1)) {
          give_up(none, abort_flag);
          break;
        }
        mbar_arrive_expect_tx(&full[stage], L::kABytes);
        uint8_t* st = smem + stage * L::kABytes;
#pragma unroll
        for (int kb = 0; kb < DP / 64; ++kb)
          tma_load_3d(st + kb * DP * 128, &tm_a, &full[stage], kb * 64, 0,
                      static_cast<int>(row_of(t)), pol);
        fills.filled(stage, phase);
      }
      fills.drain(full);
    }
  } else if (warp == L::kWarpMma) {
    // ---------------------------------------------------------------- MMA: G_t A_t
    constexpr uint32_t idesc = idesc_bf16(128, DP, false, false);
    const uint32_t g_base = smem_u32(g_tile);
    bool ok = true;
    for (int u = 0; u < n; ++u) {
      const int stage = u % L::kStages;
      const uint32_t phase = (u / L::kStages) & 1;
      if (!mbar_wait(&full[stage], phase) || !mbar_wait(g_ready, u & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (elect_one()) {
        const uint32_t a_base = smem_u32(smem + stage * L::kABytes);
#pragma unroll
        for (int ks = 0; ks < DP / 16; ++ks) {
          const uint64_t da = smem_desc_noswz(g_base + ks * 2 * 2048, 2048, 128);
          const uint64_t db = smem_desc(a_base + (ks >> 2) * DP * 128 + (ks & 3) * 32, 16, 1024);
          mma_bf16(tmem_base, da, db, idesc, ks != 0);
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
    float X[L::kCols];
    const bool first = t_hi == T;  // this launch starts at the clip's last frame
    {
      // G_{T-1} = dS_T + E_{T-1}, or G_{t_hi-1} from the previous segment
      const float* src = first ? d_state_out : carry;
      const float* ds = src ? src + bh * DD + static_cast<long>(v) * D : nullptr;
      const float* el = E_ws + row_of(T - 1) * DD;
#pragma unroll
      for (int j = 0; j < L::kCols; j += 4) {
        const int col = c0 + j;
        float4 e = make_float4(0.f, 0.f, 0.f, 0.f);
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
        if (row_ok && col < D) {
          if (first) e = __ldcg(reinterpret_cast<const float4*>(el + b4_index(v, col, D)));
          if (ds) s = __ldcg(reinterpret_cast<const float4*>(ds + col));
        }
        X[j] = s.x + e.x;
        X[j + 1] = s.y + e.y;
        X[j + 2] = s.z + e.z;
        X[j + 3] = s.w + e.w;
      }
    }
    auto pack8 = [&](int j) {
      uint4 pk;
      pk.x = pack_bf16x2(X[j], X[j + 1]);
      pk.y = pack_bf16x2(X[j + 2], X[j + 3]);
      pk.z = pack_bf16x2(X[j + 4], X[j + 5]);
      pk.w = pack_bf16x2(X[j + 6], X[j + 7]);
      return pk;
    };
    auto write_tile = [&]() {
#pragma unroll
      for (int j = 0; j < L::kCols; j += 8)
        *reinterpret_cast<uint4*>(g_tile + ((c0 + j) >> 3) * 2048 + v * 16) = pack8(j);
    };
    auto store_g = [&](int t) {  // G_t to global, bf16 s8 layout
      uint8_t* dst = reinterpret_cast<uint8_t*>(G_out + row_of(t) * DP * DP);
#pragma unroll
      for (int j = 0; j < L::kCols; j += 8)
        *reinterpret_cast<uint4*>(dst + s8_offset_bytes(v, c0 + j, DP)) = pack8(j);
    };
    auto e_slot = [&](int buf, int kg) {
      return e_buf + buf * L::kEBufBytes + (static_cast<uint32_t>(kg) * 128 + v) * 16;
    };
    // copy f (f = 0 .. n-1, while frame t_hi-2-f exists) brings E of frame t_hi-2-f into
    // buffer f % 2; one commit group per f, empty past the last copy so that the group count
    // stays uniform
    auto issue_e = [&](int f) {
      if (f < n && t_hi - 2 - f >= 0 && row_ok) {
        const float* em = E_ws + row_of(t_hi - 2 - f) * DD;
#pragma unroll
        for (int j = 0; j < L::kCols; j += 4) {
          const int col = c0 + j;
          if (col < D) cp_async16(e_slot(f & 1, col >> 2), em + b4_index(v, col, D));
        }
      }
      cp_async_commit();
    };
    issue_e(0);
    issue_e(1);
    write_tile();
    fence_async_smem();
    tc_fence_before();
    __syncwarp();  // the warp's tile writes and fences first
    if (lane == 0) mbar_arrive(g_ready);
    if (first) store_g(T - 1);  // (a later segment's G_{t_hi-1} was stored by the previous one)

    // gamma_t, beta_t of frames t_hi-1-(32*blk + lane), shuffled from lane u % 32 at step u
    const long gb_base = static_cast<long>(b) * T * p.H + h;
    auto load_gb = [&](int blk, float& gv, float& bv) {
      const int f = t_hi - 1 - (blk * 32 + static_cast<int>(lane));
      gv = f >= t_lo ? __ldg(gamma + gb_base + static_cast<long>(f) * p.H) : 0.f;
      bv = f >= t_lo ? __ldg(beta + gb_base + static_cast<long>(f) * p.H) : 0.f;
    };
    float g_cur, b_cur, g_next, b_next;
    load_gb(0, g_next, b_next);
    bool ok = true;
    for (int u = 0; u < n; ++u) {
      const int t = t_hi - 1 - u;
      if ((u & 31) == 0) {
        g_cur = g_next;
        b_cur = b_next;
        load_gb((u >> 5) + 1, g_next, b_next);
      }
      const float g = __shfl_sync(0xffffffffu, g_cur, u & 31);
      const float be = __shfl_sync(0xffffffffu, b_cur, u & 31);
      if (!mbar_wait(mma_done, u & 1)) {
        ok = false;
        break;
      }
      cp_async_wait<1>();  // copy u (E_{t-1}) has landed; copy u+1 may be in flight
      tc_fence_after();
      const bool has_e = t >= 1;
      const float gbe = g * be;
#pragma unroll
      for (int c = 0; c < L::kCols; c += 16) {
        float P[16];
        tmem_ld16(taddr + c, P);
#pragma unroll
        for (int j = 0; j < 16; j += 4) {
          const int col = c0 + c + j;
          float4 ev = make_float4(0.f, 0.f, 0.f, 0.f);
          if (has_e && row_ok && col < D)
            ev = *reinterpret_cast<const float4*>(e_slot(u & 1, col >> 2));
          X[c + j] = fmaf(g, X[c + j], fmaf(-gbe, P[j], ev.x));
          X[c + j + 1] = fmaf(g, X[c + j + 1], fmaf(-gbe, P[j + 1], ev.y));
          X[c + j + 2] = fmaf(g, X[c + j + 2], fmaf(-gbe, P[j + 2], ev.z));
          X[c + j + 3] = fmaf(g, X[c + j + 3], fmaf(-gbe, P[j + 3], ev.w));
        }
      }
      if (has_e) {
        // X = G_{t-1}: the operand of the next step's MMA (with A_{t-1}), unless t = t_lo
        if (u + 1 < n) {
          write_tile();
          fence_async_smem();
          tc_fence_before();
          __syncwarp();  // the warp's tile writes and fences first
          if (lane == 0) mbar_arrive(g_ready);
        }
        store_g(t - 1);
      }
      issue_e(u + 2);  // buffer u % 2 is free (this thread read its own slice above)
    }
    cp_async_wait<0>();
    if (!ok) give_up(none, abort_flag);
    // X = dS_0 after the first frame's step, or G_{t_lo-1} for the next segment
    float* const x_dst = t_lo == 0 ? d_state_in : carry;
    if (ok && x_dst != nullptr && row_ok) {
      float* so = x_dst + bh * DD + static_cast<long>(v) * D;
#pragma unroll
      for (int j = 0; j < L::kCols; j += 4)
        if (c0 + j < D)
          *reinterpret_cast<float4*>(so + c0 + j) = make_float4(X[j], X[j + 1], X[j + 2], X[j + 3]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == L::kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

}  // namespace gdn
