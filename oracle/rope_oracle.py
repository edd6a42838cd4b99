"""fp64 CPU oracle for the 3D rotary position embedding (RoPE) applied to q and k before the
attention layers.

TEST INFRASTRUCTURE. Only the tests may import this module; no CUDA code shares anything with
it. It is a plain float64 numpy restatement, one axis of positions at a time.

Source: the transcript of the ICLR 2026 oral talk "SANA-Video: Efficient Video Generation with
Block Linear Diffusion Transformer" introduces a 3D RoPE for the linear attention, to improve
temporal modelling. The pages give no formula, no split of the head dimension and no base, and
they do not say whether SANA-WM's GDN blocks use it.

Reading adopted, per token of frame t at latent grid cell (row, col) = (n // grid_w, n % grid_w),
for every head:
* the head dimension D splits into three contiguous even slices: d_t for time, then d_h for rows,
  then d_w for columns, with d_h = d_w = 2 * floor(D / 6) and d_t = D - 2 * d_h (the time slice
  takes the remainder);
* in the slice of axis a with width d_a, consecutive pairs (x_{2i}, x_{2i+1}), i = 0 .. d_a/2 - 1,
  rotate by the angle pos_a * theta_i, with theta_i = base ** (-2 i / d_a) (the rotary
  embedding's frequency ladder per axis, base 10000 by default);
* pos_t = t + t_offset (the absolute frame index, so streaming steps continue a clip),
  pos_h = row, pos_w = col;
* the rotation is (x, y) -> (x cos a - y sin a, x sin a + y cos a).

Parity status: pinned by ``tests/test_rope_oracle.py``. The pins are a hand-worked example,
norm preservation, the identity at position zero, invariance of the q.k products to a common
shift of positions along each axis, and the slice boundaries. Planted mistakes each fail a pin.
"""
from __future__ import annotations

import numpy as np

__all__ = ["rope_3d", "rope_3d_split"]


def rope_3d_split(D: int):
    """(d_t, d_h, d_w) of the reading above."""
    if D < 6 or D % 2:
        raise ValueError("D must be even and >= 6")
    d_h = 2 * (D // 6)
    return D - 2 * d_h, d_h, d_h


def _rotate(x, pos, d_a, base):
    """Rotate the pairs of slice x [..., d_a] by pos [...] * base^(-2i/d_a)."""
    i = np.arange(d_a // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / d_a)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * theta
    c, s = np.cos(ang), np.sin(ang)
    xe, xo = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = xe * c - xo * s
    out[..., 1::2] = xe * s + xo * c
    return out


def rope_3d(x, grid_h: int, grid_w: int, base: float = 10000.0, t_offset: int = 0):
    """3D RoPE of x [B, T, N, H, D] with N = grid_h * grid_w tokens per frame (row-major over
    the latent grid). Returns float64 [B, T, N, H, D]."""
    x = np.asarray(x, dtype=np.float64)
    B, T, N, H, D = x.shape
    if grid_h * grid_w != N:
        raise ValueError("grid_h * grid_w must equal N")
    d_t, d_h, d_w = rope_3d_split(D)
    t = np.arange(T, dtype=np.float64) + t_offset
    n = np.arange(N)
    row, col = (n // grid_w).astype(np.float64), (n % grid_w).astype(np.float64)
    # positions broadcast over [B, T, N, H]
    pos_t = np.broadcast_to(t[None, :, None, None], (B, T, N, H))
    pos_h = np.broadcast_to(row[None, None, :, None], (B, T, N, H))
    pos_w = np.broadcast_to(col[None, None, :, None], (B, T, N, H))
    out = np.empty_like(x)
    out[..., :d_t] = _rotate(x[..., :d_t], pos_t, d_t, base)
    out[..., d_t:d_t + d_h] = _rotate(x[..., d_t:d_t + d_h], pos_h, d_h, base)
    out[..., d_t + d_h:] = _rotate(x[..., d_t + d_h:], pos_w, d_w, base)
    return out
