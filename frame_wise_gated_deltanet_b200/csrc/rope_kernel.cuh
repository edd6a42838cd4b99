// 3D rotary position embedding (RoPE) of q or k, [B, T, N, H, D] bf16, before the attention
// layers. The SANA-Video talk introduces a 3D RoPE for its linear attention and gives no formula.
// Reading: the head dimension splits into three even slices, time (d_t), grid rows (d_h) and
// grid columns (d_w), with d_h = d_w = 2 * floor(D / 6) and the remainder to time. In each
// slice, the pairs (x_{2i}, x_{2i+1}) rotate by pos * base^(-2i / d_slice), where pos is the
// frame index (plus t_offset), the row n / grid_w or the column n % grid_w of the token.
//
// Standalone pass (gdn_rope_3d), two launches. A table kernel computes (cos, sin) of every
// (axis, position, pair) once, in double precision: T * d_t/2 + grid_h * d_h/2 + grid_w * d_w/2
// entries, about 180 KB for the 720p clip, which stay in L2. The rotation kernel then streams the
// tensor in 16-byte vectors (8 dims of one token and head), reads each pair's (cos, sin) from the
// table, rotates in f32 and rounds to bf16. It is HBM-bound: every element is read and written
// once. Each thread reads and writes the same 16 bytes, so x and y may be the same memory.
//
// Fused prologue (gdn_frame_forward_rope): the same table, and rope_rotate_tile applied by
// transform warps to the K tiles of the statistics kernel and the Q tiles of the output kernel in
// shared memory, so q and k are rotated on their way to the tensor cores and never rewritten.
#pragma once
#include "common.cuh"

namespace gdn {

struct RopeDims {
  int B, T, N, H, D;
  int grid_w;
  int d_t, d_h, d_w;
  int off_h, off_w;  // first table entry of the row / column axis
};

__global__ void __launch_bounds__(256)
    gdn_rope_table_kernel(float2* __restrict__ tab, RopeDims r, int t_offset, double log2_base) {
  const int nt = r.T * (r.d_t / 2);
  const int n_all = r.off_w + r.grid_w * (r.d_w / 2);
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n_all) return;
  int pos, i, da;
  if (e < nt) {
    pos = e / (r.d_t / 2) + t_offset;
    i = e % (r.d_t / 2);
    da = r.d_t;
  } else if (e < r.off_w) {
    const int f = e - r.off_h;
    pos = f / (r.d_h / 2);
    i = f % (r.d_h / 2);
    da = r.d_h;
  } else {
    const int f = e - r.off_w;
    pos = f / (r.d_w / 2);
    i = f % (r.d_w / 2);
    da = r.d_w;
  }
  const double theta = exp2(-(2.0 * i / da) * log2_base);
  double s, c;
  sincos(static_cast<double>(pos) * theta, &s, &c);
  tab[e] = make_float2(static_cast<float>(c), static_cast<float>(s));
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
    gdn_rope_kernel(const __nv_bfloat16* x, __nv_bfloat16* y, const float2* __restrict__ tab,
                    RopeDims r) {
  const int bt = blockIdx.x;
  const int t = bt % r.T;
  const int per_row = r.D / 8;  // 16-byte vectors per (token, head)
  const int per_tok = per_row * r.H;
  const int n0 = blockIdx.y * kRopeTokens;
  const int n1 = min(r.N, n0 + kRopeTokens);
  const long frame0 = static_cast<long>(bt) * r.N * per_tok;
  const uint4* src = reinterpret_cast<const uint4*>(x) + frame0;
  uint4* dst = reinterpret_cast<uint4*>(y) + frame0;
  const int pt = r.d_t / 2, ph = r.d_h / 2;
  for (int li = threadIdx.x; li < per_tok; li += blockDim.x) {
    const int dg = li % per_row;
    int row = n0 / r.grid_w;
    int col = n0 - row * r.grid_w;
    // the 4 pairs of this vector: axis (0 time, 1 row, 2 column) and index within the axis; the
    // (cos, sin) of time pairs (fixed for the frame) and of row pairs (fixed along a grid row)
    // are held in registers, only the column pairs' are read for every token
    int axis[4], idx[4];
    float2 cs_fix[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int j = dg * 4 + p;  // pair index over the head dimension
      axis[p] = j < pt ? 0 : (j < pt + ph ? 1 : 2);
      idx[p] = axis[p] == 0 ? j : (axis[p] == 1 ? j - pt : j - pt - ph);
      cs_fix[p] = axis[p] == 0   ? __ldg(tab + t * pt + idx[p])
                  : axis[p] == 1 ? __ldg(tab + r.off_h + row * ph + idx[p])
                                 : make_float2(1.f, 0.f);
    }
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
          __nv_bfloat162* p2 = reinterpret_cast<__nv_bfloat162*>(&raw[u]);
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const float2 cs = axis[p] == 2 ? __ldg(tab + r.off_w + col * ph + idx[p]) : cs_fix[p];
            const float2 v = __bfloat1622float2(p2[p]);
            p2[p] = __floats2bfloat162_rn(v.x * cs.x - v.y * cs.y, v.x * cs.y + v.y * cs.x);
          }
          __stcs(dst + static_cast<long>(nb + u) * per_tok + li, raw[u]);
        }
        if (++col == r.grid_w) {
          col = 0;
          ++row;
          if (nb + u + 1 < n1)  // a next token exists: the new row's pairs
#pragma unroll
            for (int p = 0; p < 4; ++p)
              if (axis[p] == 1) cs_fix[p] = __ldg(tab + r.off_h + row * ph + idx[p]);
        }
      }
    }
  }
}

// The same rotation applied in shared memory by the forward's statistics (K) and output (Q)
// kernels to a bf16 operand tile just loaded by TMA: `rows` token rows (token n0 + r in row r, all
// of frame t), each DP/8 16-byte chunks of 8 dims (chunk c in box c / 8; a box is 128 rows of
// 128 B, 128B-swizzled, kBoxBytes apart). Dims at or past D are left alone (TMA zero fill).
// Thread tid of nthreads owns chunk c = tid % (DP/8) of rows tid / (DP/8), + nthreads / (DP/8),
// ...: its 4 pairs, hence their axes and the time pairs' (cos, sin), are fixed for the tile; a
// warp covers whole rows, so its shared-memory accesses take the minimum number of wavefronts
// and its table reads for one token fall in a few adjacent sectors. The arithmetic and the
// rounding are those of gdn_rope_kernel.
template <int DP>
__device__ __forceinline__ void rope_rotate_tile(uint8_t* tile, int tid, int nthreads, int rows,
                                                 int n0, int t, int D, const RopeArgs& ra) {
  constexpr int kChunks = DP / 8;
  const int c = tid % kChunks;
  if (c * 8 >= D) return;
  const int r_step = nthreads / kChunks;
  int r = tid / kChunks;
  if (r >= rows) return;
  // pair p of the chunk: (cos, sin) if on the time axis, else its table offset without the
  // token's row (rg * ph) or column (cg * ph) term
  float2 ct[4];
  int off[4], axis[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int j = 4 * c + p;
    axis[p] = j < ra.pt ? 0 : (j < ra.pt + ra.ph ? 1 : 2);
    off[p] = axis[p] == 1 ? ra.off_h + j - ra.pt : ra.off_w + j - ra.pt - ra.ph;
    ct[p] = axis[p] == 0 ? __ldg(ra.tab + t * ra.pt + j) : make_float2(1.f, 0.f);
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
  auto rotate = [&](int row, const float2* cs) {
    // 128B swizzle: the chunk's 16-byte slot in its 128-byte row is c % 8 XOR row % 8
    uint4* ptr = reinterpret_cast<uint4*>(box + row * 128 + (((c & 7) ^ (row & 7)) << 4));
    uint4 raw = *ptr;
    __nv_bfloat162* p2 = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const float2 v = __bfloat1622float2(p2[p]);
      p2[p] = __floats2bfloat162_rn(v.x * cs[p].x - v.y * cs[p].y, v.x * cs[p].y + v.y * cs[p].x);
    }
    *ptr = raw;
  };
  // two rows at a time: both rows' table reads are in flight together
  for (; r < rows; r += 2 * r_step) {
    const bool second = r + r_step < rows;
    int rg2 = rg, cg2 = cg;
    advance(rg2, cg2);
    float2 cs[8];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      cs[p] = axis[p] == 0 ? ct[p] : __ldg(ra.tab + off[p] + (axis[p] == 1 ? rg : cg) * ra.ph);
      cs[4 + p] = axis[p] == 0 || !second
                      ? ct[p]
                      : __ldg(ra.tab + off[p] + (axis[p] == 1 ? rg2 : cg2) * ra.ph);
    }
    rotate(r, cs);
    if (second) rotate(r + r_step, cs + 4);
    rg = rg2;
    cg = cg2;
    advance(rg, cg);
  }
}

}  // namespace gdn
