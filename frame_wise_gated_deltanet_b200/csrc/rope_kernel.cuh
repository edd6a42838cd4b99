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
// Fused prologue (gdn_frame_forward_rope): the same table, and rope_rotate_row applied by
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

// x, y: [B, T, N, H, D] bf16 (may be the same memory). Grid (B*T, chunks): blockIdx.x is one
// frame of one batch element, whose N*H*D/8 16-byte vectors (frame_vecs) the blockIdx.y chunks
// cover; all index arithmetic is 32-bit and the frame index is per block. Each thread loads
// kRopeVecs vectors (a block's stride apart, so a warp's accesses stay coalesced) before it
// rotates and stores any of them: several loads in flight per thread. It reads and writes only
// its own vectors, so in place is safe.
constexpr int kRopeVecs = 4;

__device__ __forceinline__ void rope_rotate_vec(uint4& raw, int vi, int per_tok, int per_row,
                                                const float2* __restrict__ tab,
                                                const float2* __restrict__ tab_t,
                                                const RopeDims& r) {
  const int n = vi / per_tok;
  const int dg = (vi - n * per_tok) % per_row;
  const int row = n / r.grid_w;
  const int col = n - row * r.grid_w;
  __nv_bfloat162* p2 = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int d = dg * 8 + 2 * p;  // first dim of the pair (slices have even widths)
    float2 cs;
    if (d < r.d_t)
      cs = tab_t[d / 2];
    else if (d < r.d_t + r.d_h)
      cs = tab[r.off_h + row * (r.d_h / 2) + (d - r.d_t) / 2];
    else
      cs = tab[r.off_w + col * (r.d_w / 2) + (d - r.d_t - r.d_h) / 2];
    const float2 v = __bfloat1622float2(p2[p]);
    p2[p] = __floats2bfloat162_rn(v.x * cs.x - v.y * cs.y, v.x * cs.y + v.y * cs.x);
  }
}

__global__ void __launch_bounds__(256)
    gdn_rope_kernel(const __nv_bfloat16* x, __nv_bfloat16* y, const float2* __restrict__ tab,
                    RopeDims r, int frame_vecs) {
  const int bt = blockIdx.x;
  const int t = bt % r.T;
  const int per_row = r.D / 8;  // 16-byte vectors per (token, head)
  const int per_tok = per_row * r.H;
  const long frame0 = static_cast<long>(bt) * frame_vecs;
  const uint4* src = reinterpret_cast<const uint4*>(x) + frame0;
  uint4* dst = reinterpret_cast<uint4*>(y) + frame0;
  const float2* tab_t = tab + t * (r.d_t / 2);
  const int span = kRopeVecs * blockDim.x;  // vectors one block handles per round
  for (int v0 = blockIdx.y * span + threadIdx.x; v0 < frame_vecs; v0 += gridDim.y * span) {
    uint4 raw[kRopeVecs];
#pragma unroll
    for (int u = 0; u < kRopeVecs; ++u) {
      const int vi = v0 + u * blockDim.x;
      if (vi < frame_vecs) raw[u] = __ldcs(src + vi);
    }
#pragma unroll
    for (int u = 0; u < kRopeVecs; ++u) {
      const int vi = v0 + u * blockDim.x;
      if (vi < frame_vecs) {
        rope_rotate_vec(raw[u], vi, per_tok, per_row, tab, tab_t, r);
        __stcs(dst + vi, raw[u]);
      }
    }
  }
}

// The same rotation applied in shared memory by the forward's statistics (K) and output (Q)
// kernels to one token row of a bf16 operand tile just loaded by TMA: the 64 dims of box `box`
// (each box is 128 rows of 128 B, 128B-swizzled, kBoxBytes apart) of row `row`, which holds
// token n of frame t. Dims at or past D are left alone (TMA zero fill). The arithmetic and the
// rounding are those of gdn_rope_kernel, so the operand equals the standalone pass's output.
__device__ __forceinline__ void rope_rotate_row(uint8_t* tile, int row, int box, int n, int t,
                                                int D, const RopeArgs& ra) {
  const int rg = n / ra.grid_w;
  const int cg = n - rg * ra.grid_w;
  const int tb = t * ra.pt;                            // index of time pair 0
  const int rb = ra.off_h + rg * ra.ph - ra.pt;        // + j: row pair j - pt
  const int cb = ra.off_w + cg * ra.ph - ra.pt - ra.ph;  // + j: column pair j - pt - ph
  uint8_t* rp = tile + box * kBoxBytes + row * 128;
  const uint32_t sw = row & 7;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const int d0 = box * 64 + c * 8;
    if (d0 >= D) break;
    uint4* ptr = reinterpret_cast<uint4*>(rp + ((c ^ sw) << 4));
    uint4 raw = *ptr;
    __nv_bfloat162* p2 = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int j = (d0 >> 1) + i;  // pair index over the head dimension
      const int e = j < ra.pt ? tb + j : (j < ra.pt + ra.ph ? rb + j : cb + j);
      const float2 cs = __ldg(ra.tab + e);
      const float2 v = __bfloat1622float2(p2[i]);
      p2[i] = __floats2bfloat162_rn(v.x * cs.x - v.y * cs.y, v.x * cs.y + v.y * cs.x);
    }
    *ptr = raw;
  }
}

}  // namespace gdn
