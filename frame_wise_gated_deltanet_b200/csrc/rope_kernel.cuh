// 3D rotary position embedding (RoPE) of q or k, [B, T, N, H, D] bf16, before the attention
// layers. The SANA-Video talk introduces a 3D RoPE for its linear attention and gives no formula.
// Reading: the head dimension splits into three even slices, time (d_t), grid rows (d_h) and
// grid columns (d_w), with d_h = d_w = 2 * floor(D / 6) and the remainder to time. In each
// slice, the pairs (x_{2i}, x_{2i+1}) rotate by pos * base^(-2i / d_slice), where pos is the
// frame index (plus t_offset), the row n / grid_w or the column n % grid_w of the token.
//
// Two launches. A table kernel computes (cos, sin) of every (axis, position, pair) once, in
// double precision: T * d_t/2 + grid_h * d_h/2 + grid_w * d_w/2 entries, about 180 KB for the
// 720p clip, which stay in L2. The rotation kernel then streams the tensor in 16-byte vectors (8
// dims of one token and head), reads each pair's (cos, sin) from the table, rotates in f32 and
// rounds to bf16. It is HBM-bound: every element is read and written once. Each thread reads and
// writes the same 16 bytes, so x and y may be the same memory.
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

// x, y: [B, T, N, H, D] bf16 (may be the same memory); n_vec = B*T*N*H*D/8.
__global__ void __launch_bounds__(256)
    gdn_rope_kernel(const __nv_bfloat16* x, __nv_bfloat16* y, const float2* __restrict__ tab,
                    RopeDims r, long n_vec) {
  const int per_row = r.D / 8;  // 16-byte vectors per (token, head)
  const long stride = static_cast<long>(gridDim.x) * blockDim.x;
  for (long vi = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x; vi < n_vec;
       vi += stride) {
    const int dg = static_cast<int>(vi % per_row);
    const long tok = vi / per_row / r.H;  // (b*T + t)*N + n
    const int n = static_cast<int>(tok % r.N);
    const int t = static_cast<int>((tok / r.N) % r.T);
    const int row = n / r.grid_w;
    const int col = n - row * r.grid_w;
    uint4 raw = __ldcs(reinterpret_cast<const uint4*>(x) + vi);
    __nv_bfloat162* p2 = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const int d = dg * 8 + 2 * p;  // first dim of the pair (slices have even widths)
      float2 cs;
      if (d < r.d_t)
        cs = tab[t * (r.d_t / 2) + d / 2];
      else if (d < r.d_t + r.d_h)
        cs = tab[r.off_h + row * (r.d_h / 2) + (d - r.d_t) / 2];
      else
        cs = tab[r.off_w + col * (r.d_w / 2) + (d - r.d_t - r.d_h) / 2];
      const float2 v = __bfloat1622float2(p2[p]);
      p2[p] = __floats2bfloat162_rn(v.x * cs.x - v.y * cs.y, v.x * cs.y + v.y * cs.x);
    }
    __stcs(reinterpret_cast<uint4*>(y) + vi, raw);
  }
}

}  // namespace gdn
