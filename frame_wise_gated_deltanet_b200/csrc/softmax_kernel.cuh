// Chunk-causal softmax attention of the hybrid DiT's softmax blocks (the ai-papers.net SANA-WM
// article, section "ハイブリッドアテンション機構", and the gen-hub.ru article, section
// "Архитектура: четыре нетривиальных решения": softmax attention in blocks 3, 7, 11, 15 and 19;
// the gen-hub.ru section "Три режима на любой вкус": a bidirectional and chunk-causal
// autoregressive modes). Per head, over the clip's L = T*N tokens (token r = t*N + n):
//
//     O = softmax(Q K^T * scale + M) V,  M[r, r'] = 0 if frame(r') < (chunk(r) + 1) * F, else -inf
//
// with chunk(r) = frame(r) / F: bidirectional inside a chunk of F frames, causal across chunks
// (F >= T: fully bidirectional).
//
// One persistent CTA per SM takes work items (b, h, 128-query tile) from a global counter in the
// order of softmax_item, and walks the key tiles the tile's queries may see (128 keys each, up to the chunk limit
// of its last query) with an online softmax:
//   S_j = Q K_j^T                       tcgen05, Q and K_j K-major from 128B-swizzled TMA tiles,
//                                       into one of two TMEM buffers (128 columns each)
//   m = max(m, rowmax(S_j) * c), P_j = 2^(S_j * c - m), l = l * 2^(m_old - m) + rowsum(P_j)
//   O = O * 2^(m_old - m) + P_j V_j     tcgen05, P_j (bf16) K-major from shared memory, V_j MN-major
//                                       straight from its TMA tile, O accumulated in TMEM
// with c = scale * log2(e). The running maximum used for P is only raised when a row's maximum
// grows by more than 8 (log2 units, so P <= 2^8): O is then rescaled in TMEM by the softmax
// warps, and otherwise left alone (P and l use the same stale maximum, so O / l is unchanged).
// At the end of an item O / l is converted to bf16 in the Q tile's buffer and TMA-stored.
//
// Warp roles (10 warps): warp 0 TMA producer (Q once per item, K and V tiles through separate
// 2-stage rings), warp 1 TMEM allocator + MMA issuer (S_{j+1} is issued before PV_j so the tensor
// core computes the next scores while the softmax works on these), warps 2..9 softmax and
// epilogue (two threads per query row, each with half of the row's keys and of O's columns: TMEM
// lane = row; the halves combine their maxima and sums through spare TMEM columns). Every wait
// is bounded (GDN_ERR_TIMEOUT).
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace gdn {

template <int DP>
struct SoftmaxLayout {
  static constexpr int kBoxes = DP / 64;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;  // 128 rows x DP bf16
  static constexpr int kPBytes = 2 * kBoxBytes;          // 128 queries x 128 keys bf16
  static constexpr int kStages = 2;                      // K ring and V ring depth
  static constexpr int kSoftmaxWarps = 8;               // two per TMEM lane quarter
  static constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
  static constexpr int kThreads = 64 + kSoftmaxThreads;
  static constexpr int kTmemCols = 512;                  // S buffers [0,256), O [256, 256+DP)
  static constexpr int kOCol = 256;
  static constexpr int kXCol = 256 + DP;                 // 6 columns exchanging row partials
  static constexpr int kSmemBytes =
      kTileBytes + 2 * kStages * kTileBytes + 2 * kPBytes + 512 + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

// Key limit of query token r: the tokens of every frame up to the end of r's chunk.
__device__ __forceinline__ int softmax_key_limit(int r, int N, int T, int F) {
  const int t = r / N;
  const int c = t / F;
  const int end = (c + 1) * F;
  return (end < T ? end : T) * N;
}

struct SoftmaxItem {
  int b, h, q0;
  int n_kt;     // key tiles the item walks
  int kmin;     // smallest key limit of its queries (tiles below it need no mask)
};

// Work items in the order CTAs take them from a global counter: (batch, head) pairs in groups of
// G (whose K and V together fit in L2), and inside a group the query tiles from the last (the
// most key tiles) to the first, the group's heads interleaved: the longest items start first,
// so CTAs that take the short ones last finish together, and the K and V tiles every item of a
// head re-reads stay in L2 while the group runs.
__device__ __forceinline__ SoftmaxItem softmax_item(long item, int B, int H, int T, int N, int F,
                                                    int G) {
  const int L = T * N;
  const int nqt = (L + kRowsPerTile - 1) / kRowsPerTile;
  const int BH = B * H;
  const long per_group = static_cast<long>(G) * nqt;
  const int g = static_cast<int>(item / per_group);
  const int r = static_cast<int>(item - g * per_group);
  const int ng = min(G, BH - g * G);  // heads of this group (the last may have fewer)
  const int bh = g * G + r % ng;
  const int qt = nqt - 1 - r / ng;
  SoftmaxItem it;
  it.b = bh / H;
  it.h = bh - it.b * H;
  it.q0 = qt * kRowsPerTile;
  const int last = min(it.q0 + kRowsPerTile, L) - 1;
  it.n_kt = (softmax_key_limit(last, N, T, F) + kRowsPerTile - 1) / kRowsPerTile;
  it.kmin = softmax_key_limit(it.q0, N, T, F);
  return it;
}

// tm_q, tm_k, tm_v, tm_o: 4-D maps (D, H, T*N, B) of [B, T, N, H, D] bf16, boxes 64 x 1 x 128 x 1
// (rows past T*N read as zero and are not stored). c = scale * log2(e). next_item: a zeroed
// work counter; G: (batch, head) pairs per group of softmax_item.
template <int DP>
__global__ void __launch_bounds__(SoftmaxLayout<DP>::kThreads, 1)
    gdn_softmax_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_o, int B, int H, int T, int N,
                       int F, float c, int* next_item, int G) {
  using L = SoftmaxLayout<DP>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1k(smem_raw);
  uint8_t* q_buf = smem;                                   // Q tile, then the O staging tile
  uint8_t* k_ring = q_buf + L::kTileBytes;
  uint8_t* v_ring = k_ring + L::kStages * L::kTileBytes;
  uint8_t* p_buf = v_ring + L::kStages * L::kTileBytes;    // two P tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(p_buf + 2 * L::kPBytes);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;    // [2]
  uint64_t* k_empty = bars + 4;   // [2]
  uint64_t* v_full = bars + 6;    // [2]
  uint64_t* v_empty = bars + 8;   // [2]
  uint64_t* s_full = bars + 10;   // [2] S_j in TMEM buffer j % 2
  uint64_t* s_free = bars + 12;   // [2] its scores are read (128 arrivals)
  uint64_t* p_full = bars + 14;   // [2] P_j written, O rescaled (128 arrivals)
  uint64_t* p_free = bars + 16;   // [2] PV_j complete (P buffer free, O updated)
  uint64_t* o_empty = bars + 18;  // the epilogue has read O (128 arrivals)
  uint64_t* mma_drain = bars + 19;
  // item ids from the producer to the other warps (it runs at most one item ahead: the Q buffer)
  ItemRing ring{reinterpret_cast<int*>(bars + 28), bars + 20};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ring.ids + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t warp = warp_id();
  const uint32_t lane = lane_id();
  const int Ltok = T * N;
  const int nqt = (Ltok + kRowsPerTile - 1) / kRowsPerTile;
  const long n_items = static_cast<long>(B) * H * nqt;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], L::kSoftmaxWarps);  // one arrival per softmax warp
      mbar_init(&p_full[i], L::kSoftmaxWarps);
      mbar_init(&p_free[i], 1);
    }
    mbar_init(o_empty, L::kSoftmaxWarps);
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
  auto lost = [&]() {
    record_error(kErrTimeout);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (elect_one()) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      const uint64_t pol_q = policy_evict_first();
      const uint64_t pol_kv = policy_evict_last();  // K, V are re-read by the head's other tiles
      StageFills<2> kf, vf;
      StageFills<1> qf;
      long g = 0;  // key tiles over all items of this CTA
      for (int li = 0; !*abort_flag; ++li) {
        const long item = ring.produce(li, next_item, n_items);
        if (item < 0) break;
        const SoftmaxItem it = softmax_item(item, B, H, T, N, F, G);
        if (li > 0 && !mbar_wait(q_empty, (li & 1) ^ 1)) {
          lost();
          break;
        }
        mbar_arrive_expect_tx(q_full, L::kTileBytes);
#pragma unroll
        for (int kb = 0; kb < L::kBoxes; ++kb)
          tma_load_4d(q_buf + kb * kBoxBytes, &tm_q, q_full, kb * 64, it.h, it.q0, it.b, pol_q);
        qf.filled(0, li & 1);
        bool ok = true;
        for (int j = 0; j < it.n_kt && ok; ++j, ++g) {
          const int s = static_cast<int>(g & 1);
          const uint32_t ph = static_cast<uint32_t>(g >> 1) & 1;
          if (!mbar_wait(&k_empty[s], ph ^ 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&k_full[s], L::kTileBytes);
#pragma unroll
          for (int kb = 0; kb < L::kBoxes; ++kb)
            tma_load_4d(k_ring + s * L::kTileBytes + kb * kBoxBytes, &tm_k, &k_full[s], kb * 64,
                        it.h, j * kRowsPerTile, it.b, pol_kv);
          kf.filled(s, ph);
          if (!mbar_wait(&v_empty[s], ph ^ 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&v_full[s], L::kTileBytes);
#pragma unroll
          for (int kb = 0; kb < L::kBoxes; ++kb)
            tma_load_4d(v_ring + s * L::kTileBytes + kb * kBoxBytes, &tm_v, &v_full[s], kb * 64,
                        it.h, j * kRowsPerTile, it.b, pol_kv);
          vf.filled(s, ph);
        }
        if (!ok) {
          lost();
          break;
        }
      }
      kf.drain(k_full);  // this thread's copies have landed, whatever the exit path
      vf.drain(v_full);
      qf.drain(q_full);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc_s = idesc_bf16(128, 128, false, false);  // Q K^T
    constexpr uint32_t idesc_o = idesc_bf16(128, DP, false, true);    // P V, V MN-major
    const uint32_t q_addr = smem_u32(q_buf);
    long g = 0;
    int li = 0;
    bool ok = true;
    // S_j = Q K_j^T into TMEM buffer g % 2
    auto issue_s = [&](long gg, int j) -> bool {
      const int s = static_cast<int>(gg & 1);
      const uint32_t ph = static_cast<uint32_t>(gg >> 1) & 1;
      if (!mbar_wait(&k_full[s], ph)) return false;
      if (gg >= 2 && !mbar_wait(&s_free[s], ph ^ 1)) return false;
      tc_fence_after();
      if (elect_one()) {
        const uint32_t k_addr = smem_u32(k_ring + s * L::kTileBytes);
#pragma unroll
        for (int ks = 0; ks < DP / 16; ++ks) {
          const uint32_t off = (ks >> 2) * kBoxBytes + (ks & 3) * 32;
          mma_bf16(tmem_base + s * 128, smem_desc(q_addr + off, 16, 1024),
                   smem_desc(k_addr + off, 16, 1024), idesc_s, ks != 0);
        }
        mma_commit(&k_empty[s]);
        mma_commit(&s_full[s]);
      }
      __syncwarp();
      (void)j;
      return true;
    };
    for (; ok; ++li) {
      const long item = ring.consume(li);
      if (item == -2) ok = false;
      if (item < 0) break;
      const SoftmaxItem it = softmax_item(item, B, H, T, N, F, G);
      if (!mbar_wait(q_full, li & 1)) {
        ok = false;
        break;
      }
      if (!issue_s(g, 0)) {
        ok = false;
        break;
      }
      for (int j = 0; j < it.n_kt; ++j) {
        const long gj = g + j;
        if (j + 1 < it.n_kt && !issue_s(gj + 1, j + 1)) {
          ok = false;
          break;
        }
        // O (+)= P_j V_j once P_j is written (and, for the item's first tile, once the previous
        // item's O has been read out)
        const int s = static_cast<int>(gj & 1);
        const uint32_t ph = static_cast<uint32_t>(gj >> 1) & 1;
        if (!mbar_wait(&p_full[s], ph) || !mbar_wait(&v_full[s], ph) ||
            (j == 0 && li > 0 && !mbar_wait(o_empty, (li & 1) ^ 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
          const uint32_t p_addr = smem_u32(p_buf + s * L::kPBytes);
          const uint32_t v_addr = smem_u32(v_ring + s * L::kTileBytes);
#pragma unroll
          for (int ks = 0; ks < kRowsPerTile / 16; ++ks) {
            const uint64_t da = smem_desc(p_addr + (ks >> 2) * kBoxBytes + (ks & 3) * 32, 16, 1024);
            const uint64_t db = smem_desc(v_addr + ks * 16 * 128, kBoxBytes, 1024);
            mma_bf16(tmem_base + L::kOCol, da, db, idesc_o, (j | ks) != 0);
          }
          mma_commit(&v_empty[s]);
          mma_commit(&p_free[s]);
        }
        __syncwarp();
      }
      g += it.n_kt;
    }
    if (!ok) lost();
    // every MMA issued here has completed before TMEM is released
    if (elect_one()) mma_commit(mma_drain);
    __syncwarp();
    mbar_wait(mma_drain, 0);
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    // Warp w owns TMEM lane quarter w % 4 (query rows 32*(w%4)..) and half hf of the key columns
    // of S and P (keys 64*hf..) and of the value columns of O; the two warps of a quarter combine
    // their row maxima (and at the end their row sums) through spare TMEM columns.
    const uint32_t quarter = warp & 3;
    const int hf = static_cast<int>(warp - 2) >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = tmem_base + ((quarter * 32) << 16);
    const int pair_bar = 2 + static_cast<int>(quarter);  // named barrier of the quarter's 2 warps
    const bool leader = (threadIdx.x == 64);
    const uint64_t pol_out = policy_evict_first();
    if (leader) tma_prefetch_desc(&tm_o);
    // this thread's partial of a row statistic -> the partner's, through TMEM column `col`
    auto exchange = [&](uint32_t col_mine, uint32_t col_other, float x) -> float {
      tmem_st1(lane_base + col_mine, x);
      tc_fence_before();
      named_bar(pair_bar, 64);
      tc_fence_after();
      return tmem_ld1(lane_base + col_other);
    };
    long g = 0;
    int li = 0;
    bool ok = true;
    float v[32];
    for (; ok; ++li) {
      const long item = ring.consume(li);
      if (item == -2) ok = false;
      if (item < 0) break;
      const SoftmaxItem it = softmax_item(item, B, H, T, N, F, G);
      const int r = min(it.q0 + row, Ltok - 1);  // rows past the clip take the last row's limit
      const int kmax = softmax_key_limit(r, N, T, F);
      float m_ref = -INFINITY;  // the maximum P is taken against (log2 units)
      float l = 0.f;            // this thread's half of the row sum
      for (int j = 0; j < it.n_kt; ++j) {
        const long gj = g + j;
        const int s = static_cast<int>(gj & 1);
        const uint32_t ph = static_cast<uint32_t>(gj >> 1) & 1;
        if (!mbar_wait(&s_full[s], ph)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int k0 = j * kRowsPerTile + hf * 64;  // first key of this thread's half
        const bool masked = j * kRowsPerTile + kRowsPerTile > it.kmin;  // uniform over the CTA
        // the half row's 64 scores in one TMEM read; invisible keys become -inf
        float sv[64];
        tmem_ld64(lane_base + s * 128 + hf * 64, sv);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[s]);  // S_j is read: its buffer may take S_{j+2}
        // four independent maxima (short dependency chains), then combined
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          if (masked && k0 + i >= kmax) sv[i] = -INFINITY;
          m4[i & 3] = fmaxf(m4[i & 3], sv[i]);
        }
        float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        // both halves' maxima (TMEM columns alternate with the tile's parity, so a partner that
        // is a tile ahead never overwrites a value still to be read)
        const uint32_t xc = L::kXCol + 2 * static_cast<uint32_t>(gj & 1);
        mx = fmaxf(mx, exchange(xc + hf, xc + (hf ^ 1), mx));
        const float m_new = fmaxf(m_ref, mx * c);
        const bool raise = m_new > m_ref + 8.f;  // the same in both warps of the quarter
        if (__any_sync(0xffffffffu, raise)) {
          // the warp's rows take their new maxima; O (from PV_{j-1}) is rescaled in TMEM
          const float alpha = ex2_approx(m_ref - m_new);  // 0 while m_ref is -inf
          l *= alpha;
          m_ref = m_new;
          if (j > 0) {
            const long gp = gj - 1;
            if (!mbar_wait(&p_free[gp & 1], static_cast<uint32_t>(gp >> 1) & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int cc = 0; cc < DP / 64; ++cc) {
              const uint32_t oc = L::kOCol + hf * (DP / 2) + cc * 32;
              tmem_ld32(lane_base + oc, v);
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] *= alpha;
              tmem_st32(lane_base + oc, v);
            }
          }
        }
        // P buffer s is free once PV_{j-2} (its previous reader) is complete
        if (gj >= 2 && !mbar_wait(&p_free[s], ph ^ 1)) {
          ok = false;
          break;
        }
        // P = 2^(S c - m_ref) as bf16 into box hf of the K-major swizzled P tile, l += sum
        uint8_t* prow = p_buf + s * L::kPBytes + hf * kBoxBytes + row * 128;
        const uint32_t sw = row & 7;
        float l8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // independent partial sums
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) {  // 8 chunks of 8 keys
          float pv[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            pv[i] = ex2_approx(fmaf(sv[kc * 8 + i], c, -m_ref));  // 2^-inf = 0: invisible keys
            l8[i] += pv[i];
          }
          uint4 pk;
          pk.x = pack_bf16x2(pv[0], pv[1]);
          pk.y = pack_bf16x2(pv[2], pv[3]);
          pk.z = pack_bf16x2(pv[4], pv[5]);
          pk.w = pack_bf16x2(pv[6], pv[7]);
          *reinterpret_cast<uint4*>(prow + ((kc ^ sw) << 4)) = pk;
        }
        l += ((l8[0] + l8[1]) + (l8[2] + l8[3])) + ((l8[4] + l8[5]) + (l8[6] + l8[7]));
        tc_fence_before();
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[s]);
      }
      if (!ok) break;
      // ---- epilogue: O / l -> bf16 into the Q buffer (free: every S MMA of the item is done
      // once its last PV is), then a TMA store (rows past the clip and dims past D are clipped)
      const long gl = g + it.n_kt - 1;
      if (!mbar_wait(&p_free[gl & 1], static_cast<uint32_t>(gl >> 1) & 1)) {
        ok = false;
        break;
      }
      tc_fence_after();
      l += exchange(L::kXCol + 4 + hf, L::kXCol + 4 + (hf ^ 1), l);
      const float inv_l = 1.f / l;
#pragma unroll 1
      for (int cc = 0; cc < DP / 64; ++cc) {
        const int col = hf * (DP / 2) + cc * 32;
        tmem_ld32(lane_base + L::kOCol + col, v);
#pragma unroll
        for (int j = 0; j < 32; j += 8) {
          uint4 pk;
          pk.x = pack_bf16x2(v[j] * inv_l, v[j + 1] * inv_l);
          pk.y = pack_bf16x2(v[j + 2] * inv_l, v[j + 3] * inv_l);
          pk.z = pack_bf16x2(v[j + 4] * inv_l, v[j + 5] * inv_l);
          pk.w = pack_bf16x2(v[j + 6] * inv_l, v[j + 7] * inv_l);
          *reinterpret_cast<uint4*>(q_buf + swz128_offset_bf16(row, col + j, kBoxBytes)) = pk;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_empty);
      fence_async_smem();
      named_bar(1, L::kSoftmaxThreads);
      if (leader) {
#pragma unroll
        for (int kb = 0; kb < L::kBoxes; ++kb)
          tma_store_4d(&tm_o, q_buf + kb * kBoxBytes, kb * 64, it.h, it.q0, it.b, pol_out);
        bulk_commit();
        bulk_wait_read<0>();  // the staging tile (the Q buffer) is read: the next Q may load
        mbar_arrive(q_empty);
      }
      g += it.n_kt;
    }
    if (leader) bulk_wait_all();
    if (!ok) lost();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

}  // namespace gdn
