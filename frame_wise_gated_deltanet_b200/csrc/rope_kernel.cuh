// 3D rotary position embedding (RoPE) of q or k, [B, T, N, H, D] bf16, before the attention
// layers. The SANA-Video talk introduces a 3D RoPE for its linear attention and gives no formula.
// Reading: the head dimension splits into three even slices, time (d_t), grid rows (d_h) and
// grid columns (d_w), with d_h = d_w = 2 * floor(D / 6) and the remainder to time. In each
// slice, the pairs (x_{2i}, x_{2i+1}) rotate by pos * base^(-2i / d_slice), where pos is the
// frame index (plus t_offset), the row n / grid_w or the column n % grid_w of the token.
//
// Standalone pass (gdn_rope_3d), two launches. A table kernel computes (cos, sin) of every
// (axis, position, pair) once, in double precision: one row per frame, grid row and grid column,
// each row padded to whole 16-byte pairs of entries (the RopeArgs layout), about 180 KB for the
// 720p clip, which stay in L2. The rotation kernel then streams the tensor in 16-byte vectors
// (8 dims of one token and head), reads the (cos, sin) of the vector's pairs from the table,
// rotates in f32 and rounds to bf16. It is HBM-bound: every element is read and written once.
// Each thread reads and writes the same 16 bytes, so x and y may be the same memory.
//
// Fused prologue (gdn_frame_forward_rope): the same table, and rope_rotate_tile applied by
// transform warps to the K tiles of the statistics kernel and the Q tiles of the output kernel in
// shared memory, so q and k are rotated on their way to the tensor cores and never rewritten.
#pragma once
#include <type_traits>

#include "common.cuh"

namespace gdn {

struct RopeDims {
  int B, T, N, H, D;
  int d_t, d_h, d_w;
  RopeArgs ra;  // table layout (ra.tab set by the caller once the table has memory)
};

// The table: entry e of the RopeArgs layout. Entries of a row outside its axis's slice are
// (1, 0); the others are (cos, sin) of pos * base^(-2i / d_axis) for the pair's index i within
// its slice.
__global__ void __launch_bounds__(256)
    gdn_rope_table_kernel(float2* __restrict__ tab, RopeDims r, int t_offset, double log2_base) {
  const RopeArgs& a = r.ra;
  const int n_all = a.off_w + a.grid_w * a.len_w;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n_all) return;
  int pos, j, first, da;
  if (e < a.off_h) {
    pos = e / a.len_t + t_offset;
    j = e % a.len_t;
    first = 0;
    da = r.d_t;
  } else if (e < a.off_w) {
    const int f = e - a.off_h;
    pos = f / a.len_h;
    j = a.j0_h + f % a.len_h;
    first = a.pt;
    da = r.d_h;
  } else {
    const int f = e - a.off_w;
    pos = f / a.len_w;
    j = a.j0_w + f % a.len_w;
    first = a.pt + a.ph;
    da = r.d_w;
  }
  const int i = j - first;
  if (i < 0 || i >= da / 2) {
    tab[e] = make_float2(1.f, 0.f);
    return;
  }
  const double theta = exp2(-(2.0 * i / da) * log2_base);
  double s, c;
  sincos(static_cast<double>(pos) * theta, &s, &c);
  tab[e] = make_float2(static_cast<float>(c), static_cast<float>(s));
}

// The 8 dims of chunk c (pairs 4c .. 4c + 3): each pair's axis (0 time, 1 grid row, 2 grid
// column) and the offset, in its axis's table rows, of the 16-byte entry pair (j & ~1, j | 1).
struct RopeChunk {
  int ax[4];
  int eo[4];
};

__device__ __forceinline__ RopeChunk rope_chunk(const RopeArgs& ra, int c) {
  RopeChunk k;
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int j = 4 * c + p;
    const int a = j < ra.pt ? 0 : (j < ra.pt + ra.ph ? 1 : 2);
    k.ax[p] = a;
    k.eo[p] = (j & ~1) - (a == 0 ? 0 : (a == 1 ? ra.j0_h : ra.j0_w));
  }
  return k;
}

// (cos, sin) of the chunk's pairs on axis a at position pos (frame, grid row or grid column) into
// cs; the chunk's other pairs are left alone. One 16-byte load per pair of pairs (2q, 2q + 1).
__device__ __forceinline__ void rope_fetch(const RopeArgs& ra, const RopeChunk& k, int a, int pos,
                                           float2* cs) {
  const int row =
      a == 0 ? pos * ra.len_t : (a == 1 ? ra.off_h + pos * ra.len_h : ra.off_w + pos * ra.len_w);
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const bool lo = k.ax[2 * q] == a, hi = k.ax[2 * q + 1] == a;
    // every lane loads (the row's first entries where neither pair is on the axis), so the load
    // is not under a divergent branch
    const int e = lo ? k.eo[2 * q] : (hi ? k.eo[2 * q + 1] : 0);
    const float4 v = __ldg(reinterpret_cast<const float4*>(ra.tab + row) + (e >> 1));
    if (lo) cs[2 * q] = make_float2(v.x, v.y);
    if (hi) cs[2 * q + 1] = make_float2(v.z, v.w);
  }
}

// Shared-space accesses (32-bit shared addresses) for the rotation of a tile in shared memory.
__device__ __forceinline__ uint4 rope_lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a)
               : "memory");
  return v;
}

__device__ __forceinline__ void rope_sts128(uint32_t a, const uint4& v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

__device__ __forceinline__ float2 rope_lds64(uint32_t a) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(a) : "memory");
  return v;
}

// Rotate the 4 pairs of a 16-byte chunk of bf16 (f32 arithmetic, bf16 rounding).
__device__ __forceinline__ void rope_rotate_chunk(uint4& raw, const float2* cs) {
  __nv_bfloat162* p2 = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float2 v = __bfloat1622float2(p2[p]);
    p2[p] = __floats2bfloat162_rn(v.x * cs[p].x - v.y * cs[p].y, v.x * cs[p].y + v.y * cs[p].x);
  }
}

// x, y: [B, T, N, H, D] bf16 (may be the same memory). Grid (B*T, token chunks): blockIdx.x is
// one frame of one batch element, blockIdx.y a chunk of kRopeTokens of its tokens. A token's
// H*D/8 16-byte vectors are consecutive, so thread i of a block owns vector i (and i + blockDim,
// ...) of every token of the chunk: the head-dim group of its vector, hence which axis each of
// its 4 pairs belongs to and the time pairs' (cos, sin), is fixed for the whole chunk; only the
// grid row and column advance from token to token (incrementally, no division per vector).
// Each thread reads and writes only its own vectors, so in place is safe.
constexpr int kRopeTokens = 16;
constexpr int kRopeBatch = 4;
constexpr int kRopeMaxThreads = 512;

__global__ void __launch_bounds__(kRopeMaxThreads)
    gdn_rope_kernel(const __nv_bfloat16* x, __nv_bfloat16* y, RopeDims r) {
  const RopeArgs& ra = r.ra;
  const int bt = blockIdx.x;
  const int t = bt % r.T;
  const int per_row = r.D / 8;  // 16-byte vectors per (token, head)
  const int per_tok = per_row * r.H;
  const int n0 = blockIdx.y * kRopeTokens;
  const int n1 = min(r.N, n0 + kRopeTokens);
  const long frame0 = static_cast<long>(bt) * r.N * per_tok;
  const uint4* src = reinterpret_cast<const uint4*>(x) + frame0;
  uint4* dst = reinterpret_cast<uint4*>(y) + frame0;
  for (int li = threadIdx.x; li < per_tok; li += blockDim.x) {
    const RopeChunk k = rope_chunk(ra, li % per_row);
    int row = n0 / ra.grid_w;
    int col = n0 - row * ra.grid_w;
    // the (cos, sin) of the vector's time pairs (fixed for the frame) and grid-row pairs (fixed
    // along a grid row) are held in registers; only the column pairs' are read for every token
    float2 cs_fix[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) cs_fix[p] = make_float2(1.f, 0.f);
    rope_fetch(ra, k, 0, t, cs_fix);
    rope_fetch(ra, k, 1, row, cs_fix);
    // groups of kRopeBatch tokens: the group's loads are issued before any of its stores (x and
    // y may be the same memory, so the compiler could not move a load above a store itself)
    for (int nb = n0; nb < n1; nb += kRopeBatch) {
      uint4 raw[kRopeBatch];
#pragma unroll
      for (int u = 0; u < kRopeBatch; ++u)
        if (nb + u < n1) raw[u] = __ldcs(src + static_cast<long>(nb + u) * per_tok + li);
#pragma unroll
      for (int u = 0; u < kRopeBatch; ++u) {
        if (nb + u < n1) {
          float2 cs[4] = {cs_fix[0], cs_fix[1], cs_fix[2], cs_fix[3]};
          rope_fetch(ra, k, 2, col, cs);
          rope_rotate_chunk(raw[u], cs);
          __stcs(dst + static_cast<long>(nb + u) * per_tok + li, raw[u]);
        }
        if (++col == ra.grid_w) {
          col = 0;
          ++row;
          if (nb + u + 1 < n1) rope_fetch(ra, k, 1, row, cs_fix);  // a next token exists
        }
      }
    }
  }
}

// Shared memory the forward's statistics and output roles set aside for a copy of the table's
// grid-row and grid-column entries in the bank-conflict-free layout of rope_stage_rc (256 bytes
// per grid row and per grid column: grid_h + grid_w up to 127). A larger grid is read from the
// table in global memory instead.
constexpr int kRopeSmemTabBytes = 32 * 1024;

// Where rope_rotate_tile reads the grid-row and grid-column pairs' (cos, sin).
struct RopeRc {
  const float2* p;  // the shared-memory copy, or the table from its first grid-row entry
  int smem;         // 1: p is the copy
};

// The copy in shared memory: position (grid row rg, or grid column cg) holds 32 entries, 8 for
// each pair index p of a chunk: entry p * 8 + s is pair 4 c + p of chunk c = c0 + s, c0 the first
// chunk with a pair on the axis (at most 7 of them at D <= 128). Grid rows at rg * 32, grid
// columns at grid_h * 32 + 8 + cg * 32. For a fixed p, the 16 lanes of one token (chunks c) read
// words 8 bytes apart, grid-row lanes in the first 64 bytes of a 128-byte bank line and
// grid-column lanes in the second: no two lanes of a token share a bank, and a warp's two tokens
// take the two wavefronts an 8-byte load of 32 lanes needs anyway. (The table's own layout, pair
// j of a row at j - j0, puts the lanes of a token 32 bytes apart, 2- to 4-way bank conflicts.)
// Entries of chunks' pairs off the axis hold (1, 0) and are never read.
__device__ __forceinline__ int rope_rc_entries(const RopeArgs& ra) {
  return (ra.grid_h + ra.grid_w) * 32 + 8;
}

// Fill the copy (tab_s: kRopeSmemTabBytes, 128-byte aligned) by threads tid of nthreads if it
// fits. The caller synchronises the CTA before the first read.
__device__ __forceinline__ RopeRc rope_stage_rc(float2* tab_s, const RopeArgs& ra, int tid,
                                                int nthreads) {
  if (rope_rc_entries(ra) * static_cast<int>(sizeof(float2)) > kRopeSmemTabBytes)
    return RopeRc{ra.tab + ra.off_h, 0};
  const int n = (ra.grid_h + ra.grid_w) * 32;
  for (int i = tid; i < n; i += nthreads) {
    const int pos = i >> 5, p = (i >> 3) & 3, s = i & 7;
    const bool row = pos < ra.grid_h;
    const int first = row ? ra.pt : ra.pt + ra.ph;  // the axis's first pair
    const int j = 4 * ((first >> 2) + s) + p;
    float2 v = make_float2(1.f, 0.f);
    if (j >= first && j < first + ra.ph)
      v = row ? __ldg(ra.tab + ra.off_h + pos * ra.len_h + j - ra.j0_h)
              : __ldg(ra.tab + ra.off_w + (pos - ra.grid_h) * ra.len_w + j - ra.j0_w);
    tab_s[row ? i : i + 8] = v;
  }
  return RopeRc{tab_s, 1};
}

// The same rotation applied in shared memory by the forward's statistics (K) and output (Q)
// kernels to a bf16 operand tile just loaded by TMA: `rows` token rows (token n0 + r in row r, all
// of frame t), each DP/8 16-byte chunks of 8 dims (chunk c in box c / 8; a box is 128 rows of
// 128 B, 128B-swizzled, kBoxBytes apart). Dims at or past D are left alone (TMA zero fill).
// Thread tid of nthreads owns chunk c = tid % (DP/8) of rows tid / (DP/8), + nthreads / (DP/8),
// ...: its 4 pairs, hence their axes and the time pairs' (cos, sin), are fixed for the tile; a
// warp covers whole rows, so its shared-memory accesses take the minimum number of wavefronts.
// The grid-row and column pairs' entries are read per row from rc (rope_stage_rc), one 8-byte
// load per pair with no branch around it. The arithmetic and the rounding are those of
// gdn_rope_kernel.
template <int DP>
__device__ __forceinline__ void rope_rotate_tile(uint8_t* tile, int tid, int nthreads, int rows,
                                                 int n0, int t, int D, const RopeArgs& ra,
                                                 const RopeRc& rc) {
  constexpr int kChunks = DP / 8;
  const int c = tid % kChunks;
  if (c * 8 >= D) return;
  const int r_step = nthreads / kChunks;
  int r = tid / kChunks;
  if (r >= rows) return;
  // entries of one grid row / grid column in rc.p
  const int sh = rc.smem ? 32 : ra.len_h, sw = rc.smem ? 32 : ra.len_w;
  // pair p of the chunk: (cos, sin) if on the time axis, else its entry's offset in rc.p (the
  // token's grid row or column adds rg * sh or cg * sw)
  float2 ct[4];
  int off[4], axis[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int j = 4 * c + p;
    axis[p] = j < ra.pt ? 0 : (j < ra.pt + ra.ph ? 1 : 2);
    if (rc.smem)
      off[p] = axis[p] == 1 ? p * 8 + c - (ra.pt >> 2)
                            : ra.grid_h * 32 + 8 + p * 8 + c - ((ra.pt + ra.ph) >> 2);
    else
      off[p] = axis[p] == 1 ? j - ra.j0_h : ra.off_w - ra.off_h + j - ra.j0_w;
    ct[p] = axis[p] == 0 ? __ldg(ra.tab + t * ra.len_t + j) : make_float2(1.f, 0.f);
  }
  uint8_t* const box = tile + (c >> 3) * kBoxBytes;
  int n = n0 + r;
  int rg = n / ra.grid_w;
  int cg = n - rg * ra.grid_w;
  const int drg = r_step / ra.grid_w, dcg = r_step - drg * ra.grid_w;
  auto advance = [&](int& g_r, int& g_c) {
    g_c += dcg;
    g_r += drg;
    if (g_c >= ra.grid_w) {
      g_c -= ra.grid_w;
      ++g_r;
    }
  };
  // the tile (and the table copy, when rc.smem) through shared-space loads and stores, issued in
  // program order: both rows' table entries and chunks are loaded before either is rotated
  const uint32_t box_s = smem_u32(box);
  auto slot = [&](int row) {
    // 128B swizzle: the chunk's 16-byte slot in its 128-byte row is c % 8 XOR row % 8
    return box_s + row * 128 + (((c & 7) ^ (row & 7)) << 4);
  };
  auto rows_loop = [&](auto smem_tab) {
    constexpr bool kS = decltype(smem_tab)::value;
    const uint32_t rc_s = kS ? smem_u32(rc.p) : 0u;
    auto entry = [&](int i) { return kS ? rope_lds64(rc_s + 8u * i) : __ldg(rc.p + i); };
    // two rows at a time: both rows' table reads are in flight together
    for (; r < rows; r += 2 * r_step) {
      const bool second = r + r_step < rows;
      int rg2 = rg, cg2 = cg;
      advance(rg2, cg2);
      float2 cs[8];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        cs[p] = axis[p] == 0 ? ct[p] : entry(off[p] + (axis[p] == 1 ? rg * sh : cg * sw));
        cs[4 + p] = axis[p] == 0 || !second
                        ? ct[p]
                        : entry(off[p] + (axis[p] == 1 ? rg2 * sh : cg2 * sw));
      }
      const uint32_t a0 = slot(r), a1 = slot(second ? r + r_step : r);
      uint4 x0 = rope_lds128(a0);
      uint4 x1 = second ? rope_lds128(a1) : x0;
      rope_rotate_chunk(x0, cs);
      rope_sts128(a0, x0);
      if (second) {
        rope_rotate_chunk(x1, cs + 4);
        rope_sts128(a1, x1);
      }
      rg = rg2;
      cg = cg2;
      advance(rg, cg);
    }
  };
  if (rc.smem)
    rows_loop(std::true_type{});
  else
    rows_loop(std::false_type{});
}

}  // namespace gdn
