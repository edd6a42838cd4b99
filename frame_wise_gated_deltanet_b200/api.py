"""PyTorch binding of the C ABI (argument marshalling only; every step runs in libgdn.so).

Tensors must be CUDA tensors of the dtypes and layouts ``include/gdn.h`` documents. Calls are
asynchronous on ``stream`` (default: torch's current stream of the tensors' device).
``key_scale=None`` passes 0 to the library, which then applies the layer's default key scale.
"""
from __future__ import annotations

from typing import Optional

import torch

from ._lib import LIB, GdnError, check

__all__ = ["gdn_frame_forward", "gdn_frame_forward_fp8", "gdn_frame_forward_host",
           "gdn_frame_forward_rope", "gdn_softmax_attention", "gdn_frame_forward_train",
           "gdn_frame_backward_saved", "gdn_train_saved_bytes",
           "gdn_frame_step", "gdn_frame_backward", "gdn_backward_workspace_bytes", "gdn_rope_3d", "gdn_frame_stats", "gdn_block_causal_la",
           "gdn_sync_status", "gdn_release_workspace", "gdn_workspace_bytes",
           "gdn_la_workspace_bytes", "GdnError"]


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _req(t: torch.Tensor, name: str, dtype, shape) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path exists)")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _scale(key_scale) -> float:
    """key_scale as the C ABI takes it: None becomes 0.0, which tells the library to apply the
    layer's default scale (no arithmetic here)."""
    return 0.0 if key_scale is None else float(key_scale)


def _stream(stream, device) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def gdn_frame_forward(q, k, v, gamma, beta, state_in=None, out=None, state_out=None,
                      key_scale: Optional[float] = None, stream=None, want_state: bool = True):
    """Frame-wise GDN over a clip. q, k, v: [B,T,N,H,D] bf16; gamma, beta: [B,T,H] f32;
    state_in: [B,H,D,D] f32 or None. Returns (out, state_out)."""
    B, T, N, H, D = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _req(t, name, torch.bfloat16, (B, T, N, H, D))
    _req(gamma, "gamma", torch.float32, (B, T, H))
    _req(beta, "beta", torch.float32, (B, T, H))
    if state_in is not None:
        _req(state_in, "state_in", torch.float32, (B, H, D, D))
    if out is None:
        out = torch.empty_like(q)
    _req(out, "out", torch.bfloat16, (B, T, N, H, D))
    if state_out is None and want_state:
        state_out = torch.empty((B, H, D, D), dtype=torch.float32, device=q.device)
    if state_out is not None:
        _req(state_out, "state_out", torch.float32, (B, H, D, D))
    with torch.cuda.device(q.device):
        check("gdn_frame_forward", LIB.gdn_frame_forward(
            _ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(state_in), _ptr(out),
            _ptr(state_out), B, H, T, N, D, _scale(key_scale), _stream(stream, q.device)))
    return out, state_out


def gdn_frame_forward_rope(q, k, v, gamma, beta, grid_h: int, grid_w: int,
                           rope_base: float = 10000.0, t_offset: int = 0, state_in=None,
                           out=None, state_out=None, key_scale: Optional[float] = None,
                           stream=None, want_state: bool = True):
    """gdn_frame_forward on q and k rotated by the 3D RoPE (N = grid_h * grid_w tokens per
    frame), the rotation fused into the layer's kernels. Returns (out, state_out)."""
    B, T, N, H, D = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _req(t, name, torch.bfloat16, (B, T, N, H, D))
    _req(gamma, "gamma", torch.float32, (B, T, H))
    _req(beta, "beta", torch.float32, (B, T, H))
    if state_in is not None:
        _req(state_in, "state_in", torch.float32, (B, H, D, D))
    if out is None:
        out = torch.empty_like(q)
    _req(out, "out", torch.bfloat16, (B, T, N, H, D))
    if state_out is None and want_state:
        state_out = torch.empty((B, H, D, D), dtype=torch.float32, device=q.device)
    if state_out is not None:
        _req(state_out, "state_out", torch.float32, (B, H, D, D))
    with torch.cuda.device(q.device):
        check("gdn_frame_forward_rope", LIB.gdn_frame_forward_rope(
            _ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(state_in), _ptr(out),
            _ptr(state_out), B, H, T, N, D, _scale(key_scale), int(grid_h), int(grid_w),
            float(rope_base), int(t_offset), _stream(stream, q.device)))
    return out, state_out


def _codes(t: torch.Tensor, name: str, shape) -> torch.Tensor:
    """E4M3 codes as uint8: accepts torch.uint8 or torch.float8_e4m3fn CUDA tensors."""
    if isinstance(t, torch.Tensor) and t.dtype == torch.float8_e4m3fn:
        t = t.view(torch.uint8)
    _req(t, name, torch.uint8, shape)
    return t


def gdn_frame_forward_fp8(q8, k8, v8, q_scale, k_scale, v_scale, gamma, beta, state_in=None,
                          out=None, state_out=None, key_scale: Optional[float] = None,
                          stream=None, want_state: bool = True):
    """Frame-wise GDN on E4M3 q, k, v ([B,T,N,H,D], uint8 codes or float8_e4m3fn) with scales
    [B,T,H] f32 (x = decode(x8) * x_scale[b,t,h]). Returns (out bf16, state_out)."""
    B, T, N, H, D = q8.shape
    q8, k8, v8 = (_codes(t, n, (B, T, N, H, D)) for t, n in ((q8, "q8"), (k8, "k8"), (v8, "v8")))
    for name, t in (("q_scale", q_scale), ("k_scale", k_scale), ("v_scale", v_scale),
                    ("gamma", gamma), ("beta", beta)):
        _req(t, name, torch.float32, (B, T, H))
    if state_in is not None:
        _req(state_in, "state_in", torch.float32, (B, H, D, D))
    if out is None:
        out = torch.empty((B, T, N, H, D), dtype=torch.bfloat16, device=q8.device)
    _req(out, "out", torch.bfloat16, (B, T, N, H, D))
    if state_out is None and want_state:
        state_out = torch.empty((B, H, D, D), dtype=torch.float32, device=q8.device)
    if state_out is not None:
        _req(state_out, "state_out", torch.float32, (B, H, D, D))
    with torch.cuda.device(q8.device):
        check("gdn_frame_forward_fp8", LIB.gdn_frame_forward_fp8(
            _ptr(q8), _ptr(k8), _ptr(v8), _ptr(q_scale), _ptr(k_scale), _ptr(v_scale),
            _ptr(gamma), _ptr(beta), _ptr(state_in), _ptr(out), _ptr(state_out),
            B, H, T, N, D, _scale(key_scale), _stream(stream, q8.device)))
    return out, state_out


def _req_host(t: torch.Tensor, name: str, dtype, shape) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def gdn_frame_forward_host(q, k, v, gamma, beta, state_in=None, out=None, state_out=None,
                           key_scale: Optional[float] = None, stream=None, device=None,
                           want_state: bool = True):
    """gdn_frame_forward on HOST tensors (pinned for overlap), streamed through the GPU in
    segments of frames. Asynchronous on ``stream`` of ``device`` (default: the current CUDA
    device): synchronise it before reading out / state_out. Returns (out, state_out); missing
    outputs are allocated as pinned host tensors."""
    B, T, N, H, D = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _req_host(t, name, torch.bfloat16, (B, T, N, H, D))
    _req_host(gamma, "gamma", torch.float32, (B, T, H))
    _req_host(beta, "beta", torch.float32, (B, T, H))
    if state_in is not None:
        _req_host(state_in, "state_in", torch.float32, (B, H, D, D))
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=True)
    _req_host(out, "out", torch.bfloat16, (B, T, N, H, D))
    if state_out is None and want_state:
        state_out = torch.empty((B, H, D, D), dtype=torch.float32, pin_memory=True)
    if state_out is not None:
        _req_host(state_out, "state_out", torch.float32, (B, H, D, D))
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(device):
        check("gdn_frame_forward_host", LIB.gdn_frame_forward_host(
            _ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(state_in), _ptr(out),
            _ptr(state_out), B, H, T, N, D, _scale(key_scale), _stream(stream, device)))
    return out, state_out


def gdn_frame_step(q, k, v, gamma, beta, state_in=None, out=None, state_out=None,
                   key_scale: Optional[float] = None, stream=None):
    """One streaming step. q, k, v: [B,N,H,D] bf16; gamma, beta: [B,H] f32; state_in /
    state_out: [B,H,D,D] f32 (pass the same tensor for an in-place update). Returns (out, state)."""
    B, N, H, D = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _req(t, name, torch.bfloat16, (B, N, H, D))
    _req(gamma, "gamma", torch.float32, (B, H))
    _req(beta, "beta", torch.float32, (B, H))
    if state_in is not None:
        _req(state_in, "state_in", torch.float32, (B, H, D, D))
    if out is None:
        out = torch.empty_like(q)
    _req(out, "out", torch.bfloat16, (B, N, H, D))
    if state_out is None:
        state_out = torch.empty((B, H, D, D), dtype=torch.float32, device=q.device)
    _req(state_out, "state_out", torch.float32, (B, H, D, D))
    with torch.cuda.device(q.device):
        check("gdn_frame_step", LIB.gdn_frame_step(
            _ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(state_in), _ptr(out),
            _ptr(state_out), B, H, N, D, _scale(key_scale), _stream(stream, q.device)))
    return out, state_out


def gdn_frame_backward(q, k, v, gamma, beta, d_out, state_in=None, d_state_out=None,
                       key_scale: Optional[float] = None, stream=None,
                       want_state_grad: bool = True):
    """Gradients of gdn_frame_forward for the cotangents d_out ([B,T,N,H,D] bf16) and
    d_state_out ([B,H,D,D] f32 or None). Returns (dq, dk, dv, d_gamma, d_beta, d_state_in);
    d_state_in is None when want_state_grad is False. 64 < D <= 128."""
    B, T, N, H, D = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("d_out", d_out)):
        _req(t, name, torch.bfloat16, (B, T, N, H, D))
    _req(gamma, "gamma", torch.float32, (B, T, H))
    _req(beta, "beta", torch.float32, (B, T, H))
    if state_in is not None:
        _req(state_in, "state_in", torch.float32, (B, H, D, D))
    if d_state_out is not None:
        _req(d_state_out, "d_state_out", torch.float32, (B, H, D, D))
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    d_gamma, d_beta = torch.empty_like(gamma), torch.empty_like(beta)
    d_state_in = (torch.empty((B, H, D, D), dtype=torch.float32, device=q.device)
                  if want_state_grad else None)
    with torch.cuda.device(q.device):
        check("gdn_frame_backward", LIB.gdn_frame_backward(
            _ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(state_in), _ptr(d_out),
            _ptr(d_state_out), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(d_gamma), _ptr(d_beta),
            _ptr(d_state_in), B, H, T, N, D, _scale(key_scale), _stream(stream, q.device)))
    return dq, dk, dv, d_gamma, d_beta, d_state_in


def gdn_train_saved_bytes(B, H, T, N, D) -> int:
    return int(LIB.gdn_train_saved_bytes(B, H, T, N, D))


def gdn_frame_forward_train(q, k, v, gamma, beta, state_in=None, saved=None, out=None,
                            state_out=None, key_scale: Optional[float] = None, stream=None):
    """gdn_frame_forward that also keeps, in `saved` (a uint8 CUDA tensor of
    gdn_train_saved_bytes bytes; allocated if None), what gdn_frame_backward_saved needs.
    64 < D <= 128. Returns (out, state_out, saved)."""
    B, T, N, H, D = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _req(t, name, torch.bfloat16, (B, T, N, H, D))
    _req(gamma, "gamma", torch.float32, (B, T, H))
    _req(beta, "beta", torch.float32, (B, T, H))
    if state_in is not None:
        _req(state_in, "state_in", torch.float32, (B, H, D, D))
    nbytes = gdn_train_saved_bytes(B, H, T, N, D)
    if saved is None:
        saved = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    _req(saved, "saved", torch.uint8, (nbytes,))
    if out is None:
        out = torch.empty_like(q)
    _req(out, "out", torch.bfloat16, (B, T, N, H, D))
    if state_out is None:
        state_out = torch.empty((B, H, D, D), dtype=torch.float32, device=q.device)
    _req(state_out, "state_out", torch.float32, (B, H, D, D))
    with torch.cuda.device(q.device):
        check("gdn_frame_forward_train", LIB.gdn_frame_forward_train(
            _ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(state_in), _ptr(out),
            _ptr(state_out), _ptr(saved), B, H, T, N, D, _scale(key_scale),
            _stream(stream, q.device)))
    return out, state_out, saved


def gdn_frame_backward_saved(q, k, v, gamma, beta, saved, d_out, state_in=None,
                             d_state_out=None, key_scale: Optional[float] = None, stream=None,
                             want_state_grad: bool = True):
    """gdn_frame_backward using the states gdn_frame_forward_train saved. Returns (dq, dk, dv,
    d_gamma, d_beta, d_state_in)."""
    B, T, N, H, D = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("d_out", d_out)):
        _req(t, name, torch.bfloat16, (B, T, N, H, D))
    _req(gamma, "gamma", torch.float32, (B, T, H))
    _req(beta, "beta", torch.float32, (B, T, H))
    _req(saved, "saved", torch.uint8, (gdn_train_saved_bytes(B, H, T, N, D),))
    if state_in is not None:
        _req(state_in, "state_in", torch.float32, (B, H, D, D))
    if d_state_out is not None:
        _req(d_state_out, "d_state_out", torch.float32, (B, H, D, D))
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    d_gamma, d_beta = torch.empty_like(gamma), torch.empty_like(beta)
    d_state_in = (torch.empty((B, H, D, D), dtype=torch.float32, device=q.device)
                  if want_state_grad else None)
    with torch.cuda.device(q.device):
        check("gdn_frame_backward_saved", LIB.gdn_frame_backward_saved(
            _ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta), _ptr(state_in), _ptr(saved),
            _ptr(d_out), _ptr(d_state_out), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(d_gamma),
            _ptr(d_beta), _ptr(d_state_in), B, H, T, N, D, _scale(key_scale),
            _stream(stream, q.device)))
    return dq, dk, dv, d_gamma, d_beta, d_state_in


def gdn_rope_3d(x, grid_h: int, grid_w: int, base: float = 10000.0, t_offset: int = 0,
                out=None, stream=None):
    """3D RoPE of q or k ([B,T,N,H,D] bf16, N = grid_h * grid_w). out=x rotates in place.
    Returns out."""
    B, T, N, H, D = x.shape
    _req(x, "x", torch.bfloat16, (B, T, N, H, D))
    if out is None:
        out = torch.empty_like(x)
    _req(out, "out", torch.bfloat16, (B, T, N, H, D))
    with torch.cuda.device(x.device):
        check("gdn_rope_3d", LIB.gdn_rope_3d(
            _ptr(x), _ptr(out), B, T, N, H, D, int(grid_h), int(grid_w), float(base),
            int(t_offset), _stream(stream, x.device)))
    return out


def gdn_softmax_attention(q, k, v, frames_per_chunk: int, scale: Optional[float] = None,
                          out=None, stream=None):
    """Chunk-causal softmax attention over the clip's tokens (q, k, v, out: [B,T,N,H,D] bf16;
    frames_per_chunk >= T is bidirectional). scale=None lets the library use 1/sqrt(D).
    Returns out."""
    B, T, N, H, D = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _req(t, name, torch.bfloat16, (B, T, N, H, D))
    if out is None:
        out = torch.empty_like(q)
    _req(out, "out", torch.bfloat16, (B, T, N, H, D))
    with torch.cuda.device(q.device):
        check("gdn_softmax_attention", LIB.gdn_softmax_attention(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), B, H, T, N, D, int(frames_per_chunk),
            0.0 if scale is None else float(scale), _stream(stream, q.device)))
    return out


def gdn_frame_stats(k, v, key_scale: Optional[float] = None, A_out=None, B_out=None, stream=None):
    """Per-frame statistics. Returns A [B,H,T,D,D] bf16 (s^2 K^T K) and B [B,H,T,D,D] f32
    (s V^T K)."""
    Bsz, T, N, H, D = k.shape
    _req(k, "k", torch.bfloat16, (Bsz, T, N, H, D))
    _req(v, "v", torch.bfloat16, (Bsz, T, N, H, D))
    if A_out is None:
        A_out = torch.empty((Bsz, H, T, D, D), dtype=torch.bfloat16, device=k.device)
    if B_out is None:
        B_out = torch.empty((Bsz, H, T, D, D), dtype=torch.float32, device=k.device)
    _req(A_out, "A_out", torch.bfloat16, (Bsz, H, T, D, D))
    _req(B_out, "B_out", torch.float32, (Bsz, H, T, D, D))
    with torch.cuda.device(k.device):
        check("gdn_frame_stats", LIB.gdn_frame_stats(
            _ptr(k), _ptr(v), _ptr(A_out), _ptr(B_out), Bsz, H, T, N, D, _scale(key_scale),
            _stream(stream, k.device)))
    return A_out, B_out


def gdn_block_causal_la(q, k, v, frames_per_block: int, state_in=None, z_in=None, out=None,
                        state_out=None, z_out=None, stream=None):
    """Block-causal linear attention with relu features and a normaliser. q, k, v:
    [B,T,N,H,D] bf16; state [B,H,D,D] f32 (row = key index); z [B,H,D] f32.
    Returns (out, state_out, z_out)."""
    B, T, N, H, D = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _req(t, name, torch.bfloat16, (B, T, N, H, D))
    if state_in is not None:
        _req(state_in, "state_in", torch.float32, (B, H, D, D))
    if z_in is not None:
        _req(z_in, "z_in", torch.float32, (B, H, D))
    if out is None:
        out = torch.empty_like(q)
    _req(out, "out", torch.bfloat16, (B, T, N, H, D))
    if state_out is None:
        state_out = torch.empty((B, H, D, D), dtype=torch.float32, device=q.device)
    if z_out is None:
        z_out = torch.empty((B, H, D), dtype=torch.float32, device=q.device)
    _req(state_out, "state_out", torch.float32, (B, H, D, D))
    _req(z_out, "z_out", torch.float32, (B, H, D))
    with torch.cuda.device(q.device):
        check("gdn_block_causal_la", LIB.gdn_block_causal_la(
            _ptr(q), _ptr(k), _ptr(v), _ptr(state_in), _ptr(z_in), _ptr(out), _ptr(state_out),
            _ptr(z_out), B, H, T, N, D, int(frames_per_block), _stream(stream, q.device)))
    return out, state_out, z_out


def gdn_sync_status(stream=None, device=None) -> int:
    """Synchronise the stream and return (and clear) the device status word (0 = OK)."""
    dev = device if device is not None else torch.cuda.current_device()
    with torch.cuda.device(dev):
        return int(LIB.gdn_sync_status(_stream(stream, dev)))


def gdn_release_workspace() -> None:
    LIB.gdn_release_workspace()


def gdn_workspace_bytes(B, H, T, N, D) -> int:
    return int(LIB.gdn_workspace_bytes(B, H, T, N, D))


def gdn_backward_workspace_bytes(B, H, T, N, D) -> int:
    return int(LIB.gdn_backward_workspace_bytes(B, H, T, N, D))


def gdn_la_workspace_bytes(B, H, T, D) -> int:
    return int(LIB.gdn_la_workspace_bytes(B, H, T, D))
