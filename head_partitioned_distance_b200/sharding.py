"""Head sharding of band-sparse attention across the ranks of a process group.

Every (b, h) of the method is independent: head h attends only to its own
distance band, and no step of the attention exchanges data between heads.  So
the heads of one batch can be spread over GPUs with no collective inside the
op; the only exchange is the all-to-all that a sequence-sharded model does
around it (each rank holds N / world tokens of every head before and after the
op, and all N tokens of its own heads inside it).

The work of a head is its pair count, about W (N - lo_h - W / 2) for band width
W = N / H: the nearest band (head 0) has about W N pairs and the farthest
about W^2 / 2.  Heads h and H - 1 - h together hold about W N pairs whatever h
is, so the heads are dealt out in such pairs ("Making Every Head Count",
Figure 1: the bands are contiguous and non-overlapping, nearest first).

Everything here is host-side plumbing on ``torch.distributed`` (NCCL between
GPUs); the attention inside is the CUDA band kernel of ``spa`` run on the
rank's heads with their global bands.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence

import torch
import torch.distributed as dist


# --------------------------------------------------------------------- assignment
def band_bounds(N: int, H: int):
    """Balanced Distance Partitioning bands as two lists (host integers), from
    the library's own host entry point spa_band_bounds, so the sharding and
    the kernels can never disagree on them."""
    if H < 1 or N < H:
        raise ValueError("need 1 <= H <= N")
    from . import spa  # the C-ABI library; fails loudly when it is not built
    return spa.spa_band_bounds(N, H)


def paired_heads(H: int, world: int) -> List[List[int]]:
    """Heads of each rank: the pairs (h, H - 1 - h), h < H / 2, dealt round-robin
    (pair p to rank p mod world).  Needs H divisible by 2 * world, so every rank
    holds H / world heads (H / (2 world) pairs)."""
    if world < 1 or H % (2 * world) != 0:
        raise ValueError(f"head pairing needs H divisible by 2 * world (H={H}, world={world})")
    out: List[List[int]] = [[] for _ in range(world)]
    for p in range(H // 2):
        out[p % world] += [p, H - 1 - p]
    return [sorted(hs) for hs in out]


def head_pairs(N: int, lo: int, hi: int) -> int:
    """Permitted (i, j) pairs of one head: distance delta occurs in N - delta rows."""
    return sum(max(0, N - dd) for dd in range(lo, hi))


def rank_pairs(N: int, H: int, world: int) -> List[int]:
    """Attention pairs each rank computes under paired_heads."""
    lo, hi = band_bounds(N, H)
    return [sum(head_pairs(N, lo[h], hi[h]) for h in hs) for hs in paired_heads(H, world)]


# --------------------------------------------------------------------- exchange
def _group_size(group) -> int:
    return dist.get_world_size(group)


def _rank(group) -> int:
    return dist.get_rank(group)


def seq_to_heads(x: torch.Tensor, heads: Sequence[Sequence[int]], group=None) -> torch.Tensor:
    """[B, H, N / world, d] (this rank's sequence chunk of every head) ->
    [B, H / world, N, d] (every token of this rank's heads, ascending head
    order), by one all-to-all.  ``heads[r]`` lists rank r's heads."""
    world = _group_size(group)
    B, H, n, d = x.shape
    if len(heads) != world or any(len(hs) * world != H for hs in heads):
        raise ValueError("heads must list H / world heads for each rank of the group")
    hl = H // world
    send = torch.stack([x[:, list(heads[r])] for r in range(world)]).contiguous()  # [world, B, hl, n, d]
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # chunk i holds sequence chunk i of this rank's heads
    return recv.permute(1, 2, 0, 3, 4).reshape(B, hl, world * n, d).contiguous()


def heads_to_seq(y: torch.Tensor, heads: Sequence[Sequence[int]], group=None) -> torch.Tensor:
    """Inverse of seq_to_heads: [B, H / world, N, d] -> [B, H, N / world, d]."""
    world = _group_size(group)
    B, hl, N, d = y.shape
    if N % world != 0:
        raise ValueError(f"the sequence ({N} tokens) must split evenly over the {world} ranks")
    if len(heads) != world or any(len(hs) != hl for hs in heads):
        raise ValueError("heads must list H / world heads for each rank of the group")
    n = N // world
    send = y.reshape(B, hl, world, n, d).permute(2, 0, 1, 3, 4).contiguous()  # [world, B, hl, n, d]
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    out = torch.empty((B, hl * world, n, d), dtype=y.dtype, device=y.device)
    for r in range(world):
        out[:, list(heads[r])] = recv[r]
    return out


class _SeqToHeads(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, heads, group):
        ctx.heads, ctx.group = heads, group
        return seq_to_heads(x, heads, group)

    @staticmethod
    def backward(ctx, g):
        return heads_to_seq(g.contiguous(), ctx.heads, ctx.group), None, None


class _HeadsToSeq(torch.autograd.Function):
    @staticmethod
    def forward(ctx, y, heads, group):
        ctx.heads, ctx.group = heads, group
        return heads_to_seq(y, heads, group)

    @staticmethod
    def backward(ctx, g):
        return seq_to_heads(g.contiguous(), ctx.heads, ctx.group), None, None


# --------------------------------------------------------------------- attention
AttnFn = Callable[..., torch.Tensor]  # (q, k, v, scale=..., lo=..., hi=...) -> o


def _default_attn() -> AttnFn:
    from . import spa  # the CUDA library; fails loudly when it is not built
    return spa.spattention


def local_heads_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, H: int, rank: int, world: int,
                          scale: Optional[float] = None, attn_fn: Optional[AttnFn] = None) -> torch.Tensor:
    """Attention of the heads ``paired_heads(H, world)[rank]`` held in full:
    q, k, v are [B, H / world, N, d] in ascending global head order; each runs
    with its global band."""
    N = q.shape[2]
    lo, hi = band_bounds(N, H)
    hs = paired_heads(H, world)[rank]
    fn = attn_fn or _default_attn()
    return fn(q, k, v, scale=scale, lo=[lo[h] for h in hs], hi=[hi[h] for h in hs])


def sequence_parallel_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, H: int,
                                scale: Optional[float] = None, group=None,
                                attn_fn: Optional[AttnFn] = None) -> torch.Tensor:
    """Band-sparse attention of a sequence-sharded batch: q, k, v are this
    rank's [B, H, N / world, d] chunk of the sequence (rank r holds tokens
    [r N / world, (r + 1) N / world)).  All-to-all to head shards, attention
    of the rank's heads over the whole sequence, all-to-all back; returns this
    rank's [B, H, N / world, d] of o.  Differentiable (the exchange's
    gradient is the opposite exchange)."""
    world = _group_size(group)
    rank = _rank(group)
    if q.shape[1] != H:
        raise ValueError("q, k, v hold every head of the rank's sequence chunk")
    heads = paired_heads(H, world)
    qh, kh, vh = (_SeqToHeads.apply(t, heads, group) for t in (q, k, v))
    oh = local_heads_attention(qh, kh, vh, H, rank, world, scale, attn_fn)
    return _HeadsToSeq.apply(oh, heads, group)
