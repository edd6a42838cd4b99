"""Head-sharded multi-GPU split of one clip (one process per GPU, torch.distributed plumbing).

Heads of the frame-wise GDN layer are independent: each carries its own D x D state through the
clip's frames, so a clip's B*H (batch, head) chains partition over ranks with no exchange on the
data path. Rank r owns the contiguous head range head_range(H, world, r) -- what a column-parallel
QKV projection emits on that rank as its own [B, T, N, H_r, D] tensors -- and runs the layer on
them through the C ABI. The only collective is the optional all-gather of the outputs (and final
states) when one consumer needs every head, done here over torch.distributed (NCCL on GPUs).

Nothing here computes any of the layer's arithmetic: the per-rank work is gdn_frame_forward (or
any of the library's entry points) on that rank's heads.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch


def head_range(H: int, world: int, rank: int) -> Tuple[int, int]:
    """[h0, h1) of the heads rank `rank` of `world` owns: contiguous ranges, the first H % world
    ranks one head longer (ranks beyond H get an empty range)."""
    if H < 1 or world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad split: H={H}, world={world}, rank={rank}")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def shard_heads(x: torch.Tensor, world: int, rank: int, dim: int) -> torch.Tensor:
    """The rank's heads of a full tensor (heads along `dim`), contiguous: [B,T,N,H,D] -> dim 3,
    [B,T,H] (gamma, beta) -> dim 2, [B,H,D,D] (state) -> dim 1."""
    h0, h1 = head_range(x.shape[dim], world, rank)
    return x.narrow(dim, h0, h1 - h0).contiguous()


def gather_heads(local: torch.Tensor, H: int, dim: int, group=None) -> torch.Tensor:
    """All-gather every rank's head slice (heads along `dim`) into the full tensor of H heads,
    in rank order. Ranks may own different numbers of heads: slices are padded to the largest
    range for the collective and trimmed after it."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    h0, h1 = head_range(H, world, rank)
    if local.shape[dim] != h1 - h0:
        raise ValueError(f"rank {rank} holds {local.shape[dim]} heads, owns {h1 - h0}")
    width = head_range(H, world, 0)[1]  # the largest range (rank 0 is never shorter)
    pad_shape = list(local.shape)
    pad_shape[dim] = width
    padded = local.new_zeros(pad_shape)
    padded.narrow(dim, 0, h1 - h0).copy_(local)
    parts = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(parts, padded.contiguous(), group=group)
    pieces = []
    for r in range(world):
        a, b = head_range(H, world, r)
        if b > a:
            pieces.append(parts[r].narrow(dim, 0, b - a))
    return torch.cat(pieces, dim=dim).contiguous()


def gdn_frame_forward_head_sharded(q, k, v, gamma, beta, H: int, state_in=None,
                                   key_scale: Optional[float] = None, gather: bool = True,
                                   group=None, stream=None):
    """The layer on this rank's heads of a clip whose H heads are split over the group's ranks.
    q, k, v: [B, T, N, H_r, D] bf16, gamma, beta: [B, T, H_r] f32, state_in: [B, H_r, D, D] f32
    or None -- this rank's heads (head_range(H, world, rank)). key_scale=None lets the library
    apply its default. Returns (out, state_out): the full [B, T, N, H, D] / [B, H, D, D] tensors
    when gather is True (one all-gather each), else this rank's slices."""
    import torch.distributed as dist
    from . import api
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    h0, h1 = head_range(H, world, rank)
    if q.shape[3] != h1 - h0:
        raise ValueError(f"rank {rank} holds {q.shape[3]} heads, owns {h1 - h0}")
    if h1 > h0:
        out, st = api.gdn_frame_forward(q, k, v, gamma, beta, state_in, key_scale=key_scale,
                                        stream=stream)
    else:  # more ranks than heads: nothing to compute, but the collective still needs a part
        B, T, N, _, D = q.shape
        out = q.new_empty((B, T, N, 0, D))
        st = torch.empty((B, 0, D, D), dtype=torch.float32, device=q.device)
    if not gather:
        return out, st
    return gather_heads(out, H, 3, group), gather_heads(st, H, 1, group)
