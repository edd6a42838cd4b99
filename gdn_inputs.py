"""Seeded synthetic inputs for the frame-wise Gated DeltaNet frame scan.

This module only draws random numbers and shapes them. It holds none of the
layer's arithmetic, so both the fp64 oracle (``oracle/``) and the CUDA library
(``frame_wise_gated_deltanet_b200``) can be fed from it without sharing any code
with each other.

Layouts (the ones the C ABI in ``include/gdn.h`` takes):

* ``q, k, v``  : ``[B, T, N, H, D]`` bfloat16, contiguous (token-major, as a
  DiT QKV projection emits it; frame ``t`` of head ``h`` is ``N`` rows with a
  stride of ``H*D`` elements).
* ``gamma, beta`` : ``[B, T, H]`` float32, one decay gate and one delta-rule
  strength per batch element, frame and head.
* ``state`` : ``[B, H, D, D]`` float32.

Workloads (the shapes of the SANA-WM / SANA-Streaming latent videos; no real
latents or weights exist here, so seeded Gaussian stand-ins of the same shapes
are used):

* ``tiny``   B1 H2  D32  T8   N16  (4x4 grid)
* ``480p``   B1 H32 D64  T21  N390 (15x26 grid)
* ``stream`` B16 H20 D128 N880 (22x40 grid), 64 chained single-frame steps
* ``720p``   B1 H20 D128 T961 N880 (22x40 grid), a 60 s clip
* ``la``     B2 H20 D112 T81  N390, block-causal linear attention, 3 frames/block
* ``softmax_480p`` / ``softmax_720p21``: chunk-causal softmax attention (chunks of 3 frames)
  of B1 H32 D64 T21 N390 and B1 H20 D128 T21 N880

q, k, v are N(0, 1) drawn in float32 and rounded to bfloat16 (round to nearest
even). gamma and beta are uniform in the stated ranges, drawn and kept in
float32.  A non-zero initial state is N(0, sigma^2) in float32.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, gate ranges, seed and kind."""

    name: str
    kind: str  # "gdn" (whole clip), "stream" (chained steps), "la" or "softmax"
    B: int
    H: int
    D: int
    T: int
    N: int
    gamma_range: tuple = (0.0, 0.0)
    beta_range: tuple = (0.0, 0.0)
    seed: int = 0
    state_std: float = 0.0  # 0 -> the clip starts from S_0 = 0
    steps: int = 0  # "stream": number of chained single-frame calls
    frames_per_block: int = 0  # "la": frames per causal block; "softmax": per chunk
    grid: str = ""  # latent token grid of one frame, for the record

    @property
    def key_scale(self) -> float:
        """1/sqrt(D*N) for the GDN workloads; 1 for block-causal LA (it cancels)."""
        if self.kind == "la":
            return 1.0
        return 1.0 / math.sqrt(self.D * self.N)

    @property
    def tokens_heads(self) -> int:
        """B*H*T*N: the unit of the throughput metric (per call for "stream")."""
        return self.B * self.H * self.T * self.N


WORKLOADS = {
    "tiny": Workload("tiny", "gdn", 1, 2, 32, 8, 16, (0.9, 0.999), (0.1, 0.9), seed=0,
                     grid="4x4"),
    "480p": Workload("480p", "gdn", 1, 32, 64, 21, 390, (0.9, 0.999), (0.05, 0.95), seed=1,
                     grid="15x26"),
    "stream": Workload("stream", "stream", 16, 20, 128, 1, 880, (0.95, 0.999), (0.1, 0.9),
                       seed=2, state_std=0.1, steps=64, grid="22x40"),
    "720p": Workload("720p", "gdn", 1, 20, 128, 961, 880, (0.95, 0.9999), (0.05, 0.95),
                     seed=3, grid="22x40"),
    # two heads of the 720p clip: the per-GPU slice of the 720p layer split 10 ways by head,
    # where the per-head state chain rather than HBM bounds the forward
    "720p_2h": Workload("720p_2h", "gdn", 1, 2, 128, 961, 880, (0.95, 0.9999), (0.05, 0.95),
                        seed=5, grid="22x40"),
    "la": Workload("la", "la", 2, 20, 112, 81, 390, seed=4, frames_per_block=3,
                   grid="15x26"),
    # chunk-causal softmax attention of the hybrid blocks (chunks of 3 frames): the 480p clip's
    # shape, and 21 frames of the 720p grid (its full 961 frames are quadratic in the tokens)
    "softmax_480p": Workload("softmax_480p", "softmax", 1, 32, 64, 21, 390, seed=1564,
                             frames_per_block=3, grid="15x26"),
    "softmax_720p21": Workload("softmax_720p21", "softmax", 1, 20, 128, 21, 880, seed=1628,
                               frames_per_block=3, grid="22x40"),
}


def _generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, gen: torch.Generator, device) -> torch.Tensor:
    """N(0,1) in float32, rounded to bfloat16 (round to nearest even)."""
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    return x.to(torch.bfloat16)


def uniform_f32(shape, lo: float, hi: float, gen: torch.Generator, device) -> torch.Tensor:
    """U[lo, hi) in float32."""
    u = torch.rand(shape, generator=gen, device=device, dtype=torch.float32)
    return (lo + (hi - lo) * u).to(torch.float32)


def clip_inputs(B: int, H: int, T: int, N: int, D: int, gamma_range=(0.9, 0.999),
                beta_range=(0.1, 0.9), seed: int = 0, state_std: float = 0.0,
                device="cpu") -> dict:
    """q, k, v ([B,T,N,H,D] bf16), gamma, beta ([B,T,H] f32), state ([B,H,D,D] f32 or None).

    Draw order from one generator: q, k, v, gamma, beta, state.
    """
    g = _generator(seed, device)
    q = normal_bf16((B, T, N, H, D), g, device)
    k = normal_bf16((B, T, N, H, D), g, device)
    v = normal_bf16((B, T, N, H, D), g, device)
    gamma = uniform_f32((B, T, H), gamma_range[0], gamma_range[1], g, device)
    beta = uniform_f32((B, T, H), beta_range[0], beta_range[1], g, device)
    state = None
    if state_std > 0.0:
        state = state_std * torch.randn((B, H, D, D), generator=g, device=device,
                                        dtype=torch.float32)
    return {"q": q, "k": k, "v": v, "gamma": gamma, "beta": beta, "state": state}


def cotangents(B: int, H: int, T: int, N: int, D: int, seed: int = 0, state_std: float = 0.0,
               device="cpu") -> dict:
    """Cotangents for the backward: d_out ([B,T,N,H,D] bf16, N(0,1)) and d_state_out
    ([B,H,D,D] f32, N(0, state_std^2), or None when state_std is 0). Draw order: d_out,
    d_state_out."""
    g = _generator(seed, device)
    d_out = normal_bf16((B, T, N, H, D), g, device)
    d_state = None
    if state_std > 0.0:
        d_state = state_std * torch.randn((B, H, D, D), generator=g, device=device,
                                          dtype=torch.float32)
    return {"d_out": d_out, "d_state": d_state}


def workload_inputs(w: Workload, device="cpu", step: Optional[int] = None) -> dict:
    """Inputs of a named workload.

    For "stream", ``step=None`` returns the initial state only ({"state": ...},
    seed ``w.seed``); ``step=j`` returns the j-th frame's q, k, v, gamma, beta
    with seed ``1000*w.seed + j`` and T=1.
    """
    if w.kind == "stream":
        if step is None:
            g = _generator(w.seed, device)
            st = w.state_std * torch.randn((w.B, w.H, w.D, w.D), generator=g,
                                           device=device, dtype=torch.float32)
            return {"state": st}
        return clip_inputs(w.B, w.H, 1, w.N, w.D, w.gamma_range, w.beta_range,
                           seed=1000 * w.seed + step, device=device)
    if w.kind in ("la", "softmax"):
        g = _generator(w.seed, device)
        shape = (w.B, w.T, w.N, w.H, w.D)
        return {"q": normal_bf16(shape, g, device), "k": normal_bf16(shape, g, device),
                "v": normal_bf16(shape, g, device), "state": None, "z": None}
    return clip_inputs(w.B, w.H, w.T, w.N, w.D, w.gamma_range, w.beta_range, seed=w.seed,
                       state_std=w.state_std, device=device)


def quantize_e4m3(x):
    """8-bit E4M3 codes of x [B, T, N, H, D] with one absmax scale per (batch, frame, head):
    scale = max |x| / 448 over the frame's tokens and dims (1 for an all-zero slice), codes =
    x / scale rounded to nearest even by torch's float8_e4m3fn conversion. Returns (uint8 codes
    [B, T, N, H, D], f32 scales [B, T, H]) on x's device. This stands in for the projection
    that would emit fp8 activations; it is input generation, not part of the layer."""
    import torch
    xf = x.float()
    amax = xf.abs().amax(dim=(2, 4))
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    codes = (xf / scale[:, :, None, :, None]).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.contiguous()
