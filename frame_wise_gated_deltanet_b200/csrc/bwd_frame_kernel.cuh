// Per-frame part of the backward: for every (b, t, h), from S_{t-1} (the state the frame
// started from) and G_t = dL/dS_t (the backward chain's output):
//
//   W_t      = S_{t-1}^T G_t + G_t^T S_{t-1}            (D x D, symmetric)
//   W'_t     = -s * gamma_t * W_t                       (stored bf16, s8 layout, for dK)
//   dgamma_t = <G_t, S_{t-1}> - beta_t * <G_t, S_{t-1} A_t>
//   dbeta_t  = <G_t, B_t>     - gamma_t * <G_t, S_{t-1} A_t>
//
// with <G, S A> = <S^T G, A> = <W, A> / 2 (A_t symmetric), s the key scale. The key gradient
// then needs only token GEMMs: dK = s beta (V G_t + K W'_t).
//
// W_t is one tcgen05 accumulation of two 128 x 128 x 128 products whose operands are both
// MN-major: the s8 layout of a state (8 consecutive keys in 16 bytes, rows 16 bytes apart) is a
// no-swizzle core-matrix layout along either index, so S^T G reads the same tiles the forward's
// K-major GEMMs read, with LBO = 128 bytes between 8-row groups (the contraction index) and
// SBO = DP*16 bytes between 8-key groups. One item per loop iteration and CTA (4 warps,
// thread = TMEM lane = row); two CTAs per SM hide each other's load latency.
//
// Every operand arrives with one round of memory latency: S_{t-1}, G_t and A_t by bulk copies
// on one mbarrier, and each thread's row of B_t (32 float4 in the four-key interleaved layout)
// as plain loads issued before that wait. <W, A> reads A_t by columns (A_t is symmetric), so
// the 32 lanes of a warp read 64 contiguous bytes of shared memory.
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace gdn {

template <int DP>
struct BwdFrameLayout {
  static constexpr int kTileBytes = DP * DP * 2;
  static constexpr int kThreads = 128;
  static constexpr int kTmemCols = DP < 32 ? 32 : DP;
  static constexpr int kSmemBytes = 3 * kTileBytes + 256 + 1024;  // S, G, A tiles
};

// S_ws, G_ws, W_out: bf16 DP x DP per row (s8 layout), row (b*H+h)*T + t; A_ws: bf16 D x D
// row-major per row; B_ws: f32 D x D per row (b4_index layout); state_in: f32 [B*H][D][D]
// row-major (S_{-1}; nullptr = zero); d_gamma, d_beta: [B, T, H]. Items: frames [t_lo, t_hi)
// of every head.
template <int DP>
__global__ void __launch_bounds__(BwdFrameLayout<DP>::kThreads)
    gdn_bwd_frame_kernel(const __nv_bfloat16* __restrict__ S_ws,
                         const __nv_bfloat16* __restrict__ G_ws,
                         const __nv_bfloat16* __restrict__ A_ws, const float* __restrict__ B_ws,
                         const float* __restrict__ state_in, const float* __restrict__ gamma,
                         const float* __restrict__ beta, __nv_bfloat16* __restrict__ W_out,
                         float* __restrict__ d_gamma, float* __restrict__ d_beta, int t_lo,
                         int t_hi, Problem p) {
  using L = BwdFrameLayout<DP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1k(smem_raw);
  uint8_t* s_tile = smem;
  uint8_t* g_tile = smem + L::kTileBytes;
  uint8_t* a_tile = g_tile + L::kTileBytes;  // A_t, D x D bf16 row-major
  uint64_t* loaded = reinterpret_cast<uint64_t*>(a_tile + L::kTileBytes);
  uint64_t* mma_done = loaded + 1;
  uint64_t* mma_drain = mma_done + 1;  // all of this CTA's MMAs are complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_drain + 1);
  float* red = reinterpret_cast<float*>(tmem_slot + 4);  // [4 warps][3]

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int tid = threadIdx.x;
  const int T = p.T;
  const int D = p.D;
  const long DD = static_cast<long>(D) * D;
  const int nt = t_hi - t_lo;
  const long n_items = static_cast<long>(p.B) * p.H * nt;

  if (tid == 0) {
    mbar_init(loaded, 1);
    mbar_init(mma_done, 1);
    mbar_init(mma_drain, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t taddr = tmem_base + ((warp * 32) << 16);
  const int r = tid;  // TMEM lane, and the row this thread reads from the tiles and globals
  bool ok = true;

  int li = 0;
  for (long item = blockIdx.x; item < n_items && ok; item += gridDim.x, ++li) {
    const int bh = static_cast<int>(item / nt);
    const int t = t_lo + static_cast<int>(item - static_cast<long>(bh) * nt);
    const int b = bh / p.H;
    const int h = bh - b * p.H;
    const long row = static_cast<long>(bh) * T + t;
    // ------------------------------------------------ S_{t-1} and G_t into shared memory
    if (tid == 0) {
      const uint64_t pol = policy_evict_first();
      const uint32_t a_bytes = static_cast<uint32_t>(DD * 2);
      mbar_arrive_expect_tx(loaded, (t >= 1 ? 2 * L::kTileBytes : L::kTileBytes) + a_bytes);
      if (t >= 1) bulk_load(s_tile, S_ws + (row - 1) * DP * DP, L::kTileBytes, loaded, pol);
      bulk_load(g_tile, G_ws + row * DP * DP, L::kTileBytes, loaded, pol);
      bulk_load(a_tile, A_ws + row * DD, a_bytes, loaded, pol);
    }
    // this thread's row r of B_t, 4 keys per float4 (in flight while the copies land)
    float4 bq[DP / 4];
    {
      const float* bm = B_ws + row * DD;
#pragma unroll
      for (int i = 0; i < DP / 4; ++i)
        bq[i] = (r < D && i < D / 4)
                    ? __ldcs(reinterpret_cast<const float4*>(bm + b4_index(r, i * 4, D)))
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (t == 0) {
      // S_{-1} = state_in, converted to the bf16 s8 layout (row r, 8 keys per 16 bytes)
      const float* si = state_in ? state_in + static_cast<long>(bh) * DD + static_cast<long>(r) * D
                                 : nullptr;
#pragma unroll 4
      for (int kg = 0; kg < DP / 8; ++kg) {
        float x[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int k = kg * 8 + j;
          x[j] = (si != nullptr && r < D && k < D) ? si[k] : 0.f;
        }
        uint4 pk;
        pk.x = pack_bf16x2(x[0], x[1]);
        pk.y = pack_bf16x2(x[2], x[3]);
        pk.z = pack_bf16x2(x[4], x[5]);
        pk.w = pack_bf16x2(x[6], x[7]);
        *reinterpret_cast<uint4*>(s_tile + kg * (DP * 16) + r * 16) = pk;
      }
      fence_async_smem();
    }
    // a timed-out wait is decided for the whole CTA, so that every thread leaves together
    if (__syncthreads_or(!mbar_wait(loaded, li & 1))) {
      ok = false;
      if (tid == 0) mbar_wait(loaded, li & 1);  // (bounded) for the copies still in flight
      break;
    }
    // ------------------------------------------------ W_t = S^T G + G^T S (both MN-major)
    if (warp == 0) {
      tc_fence_after();
      if (elect_one()) {
        constexpr uint32_t idesc = idesc_bf16(128, DP, true, true);
        const uint32_t sb = smem_u32(s_tile), gb = smem_u32(g_tile);
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
          const uint32_t a = pass == 0 ? sb : gb;
          const uint32_t bb = pass == 0 ? gb : sb;
#pragma unroll
          for (int ks = 0; ks < DP / 16; ++ks) {
            // rows 16ks .. 16ks+15 of both tiles: two 8-row groups, 128 bytes apart
            const uint64_t da = smem_desc_noswz(a + ks * 256, 128, DP * 16);
            const uint64_t db = smem_desc_noswz(bb + ks * 256, 128, DP * 16);
            mma_bf16(tmem_base, da, db, idesc, (pass | ks) != 0);
          }
        }
        mma_commit(mma_done);
      }
      __syncwarp();
    }
    // ------------------------------------------------ <G, S> and <G, B> (row r of each)
    // (tiles are zero past D, and so is bq)
    float gs = 0.f, gb = 0.f, gsa = 0.f;
#pragma unroll
    for (int kg = 0; kg < DP / 8; ++kg) {
      const uint4 gv = *reinterpret_cast<const uint4*>(g_tile + kg * (DP * 16) + r * 16);
      const uint4 sv = *reinterpret_cast<const uint4*>(s_tile + kg * (DP * 16) + r * 16);
      const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
      const __nv_bfloat162* s2 = reinterpret_cast<const __nv_bfloat162*>(&sv);
      const float bb[8] = {bq[2 * kg].x,     bq[2 * kg].y,     bq[2 * kg].z,     bq[2 * kg].w,
                           bq[2 * kg + 1].x, bq[2 * kg + 1].y, bq[2 * kg + 1].z, bq[2 * kg + 1].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 gf = __bfloat1622float2(g2[j]);
        const float2 sf = __bfloat1622float2(s2[j]);
        gs = fmaf(gf.x, sf.x, fmaf(gf.y, sf.y, gs));
        gb = fmaf(gf.x, bb[2 * j], fmaf(gf.y, bb[2 * j + 1], gb));
      }
    }
    // ------------------------------------------------ read W row r: <W, A>, W' to global
    const bool mma_ok = mbar_wait(mma_done, li & 1);
    tc_fence_after();
    const float gam = __ldg(gamma + (static_cast<long>(b) * T + t) * p.H + h);
    const float bet = __ldg(beta + (static_cast<long>(b) * T + t) * p.H + h);
    const float wscale = -p.key_scale * gam;
    // column r of A_t (= row r: A_t is symmetric); lanes read consecutive elements
    const __nv_bfloat16* acol = reinterpret_cast<const __nv_bfloat16*>(a_tile) + r;
    uint8_t* wdst = reinterpret_cast<uint8_t*>(W_out + row * DP * DP);
#pragma unroll 1
    for (int c = 0; c < DP; c += 32) {
      float w[32];
      tmem_ld32(taddr + c, w);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (r < D && c + j < D) gsa = fmaf(w[j], __bfloat162float(acol[(c + j) * D]), gsa);
#pragma unroll
      for (int j = 0; j < 32; j += 8) {
        uint4 pk;
        pk.x = pack_bf16x2(wscale * w[j], wscale * w[j + 1]);
        pk.y = pack_bf16x2(wscale * w[j + 2], wscale * w[j + 3]);
        pk.z = pack_bf16x2(wscale * w[j + 4], wscale * w[j + 5]);
        pk.w = pack_bf16x2(wscale * w[j + 6], wscale * w[j + 7]);
        *reinterpret_cast<uint4*>(wdst + s8_offset_bytes(r, c + j, DP)) = pk;
      }
    }
    // ------------------------------------------------ reduce over the CTA
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      gs += __shfl_xor_sync(0xffffffffu, gs, off);
      gb += __shfl_xor_sync(0xffffffffu, gb, off);
      gsa += __shfl_xor_sync(0xffffffffu, gsa, off);
    }
    if (lane == 0) {
      red[warp * 3] = gs;
      red[warp * 3 + 1] = gb;
      red[warp * 3 + 2] = gsa;
    }
    tc_fence_before();
    // also: every thread is done with the tiles and TMEM of this item
    if (__syncthreads_or(!mma_ok)) {
      ok = false;
      break;
    }
    if (tid == 0) {
      float sgs = 0.f, sgb = 0.f, sgsa = 0.f;
      for (int w = 0; w < 4; ++w) {
        sgs += red[w * 3];
        sgb += red[w * 3 + 1];
        sgsa += red[w * 3 + 2];
      }
      const long gi = (static_cast<long>(b) * T + t) * p.H + h;
      const float sa = 0.5f * sgsa;  // <G_t, S_{t-1} A_t>
      d_gamma[gi] = sgs - bet * sa;
      d_beta[gi] = sgb - gam * sa;
    }
    __syncthreads();  // red[] is rewritten by the next item
  }
  if (!ok && tid == 0) record_error(kErrTimeout);

  // every MMA issued here has completed before TMEM is released
  if (warp == 0) {
    if (elect_one()) mma_commit(mma_drain);
    __syncwarp();
    mbar_wait(mma_drain, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

}  // namespace gdn
