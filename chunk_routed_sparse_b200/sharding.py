"""Multi-GPU plumbing for the head split: which (b, h) slices a rank owns, the
all-gather of the output shares, and the all-to-all re-sharding between sequence
shards and the head split.

Every stage of the method is independent per (batch, head) slice (the
jxzklqfsx.com MoC write-up, "計算效率": all operations are head-independent), so
ranks that own disjoint slice shares run the unchanged calls with no exchange on
the data path; these helpers only move inputs and outputs around it. They use
``torch.distributed`` (NCCL on GPUs, gloo on CPU) and nothing of the library.
"""
from __future__ import annotations

import torch


def shard_slices(B: int, H: int, world: int, rank: int):
    """Contiguous share [s0, s1) of the B*H flat (b, h) slices for one rank:
    every slice belongs to exactly one rank and the shares differ by at most
    one slice. Every stage of the path is independent per slice (the
    jxzklqfsx.com MoC write-up, "計算效率": all operations are
    head-independent), so the shares run with no exchange."""
    n = B * H
    base, extra = divmod(n, world)
    s0 = rank * base + min(rank, extra)
    return s0, s0 + base + (1 if rank < extra else 0)


def gather_slices(part: torch.Tensor, n_slices: int, world: int) -> torch.Tensor:
    """All-gather the per-rank slice shares ([s1 - s0, ...] each, in rank
    order) into the whole [n_slices, ...] tensor on every rank. Shares are
    padded to the largest one for the collective and trimmed after."""
    import torch.distributed as dist
    sizes = [shard_slices(1, n_slices, world, r) for r in range(world)]
    mx = max(b - a for a, b in sizes)
    buf = torch.zeros((mx,) + tuple(part.shape[1:]), dtype=part.dtype, device=part.device)
    buf[:part.shape[0]].copy_(part)
    out = torch.empty((world * mx,) + tuple(part.shape[1:]), dtype=part.dtype, device=part.device)
    dist.all_gather_into_tensor(out, buf)
    return torch.cat([out[r * mx:r * mx + (b - a)] for r, (a, b) in enumerate(sizes)])


def _bytes_view(x: torch.Tensor, lead: int) -> torch.Tensor:
    # a contiguous tensor as [its first `lead` dims..., bytes]: collectives then move
    # raw bytes (int8, which every backend supports) whatever the element type
    x = x.contiguous()
    return x.view(torch.int8).reshape(tuple(x.shape[:lead]) + (-1,))


def seq_to_heads(xs: torch.Tensor, n_slices: int, L: int, world: int, rank: int) -> torch.Tensor:
    """Re-shard sequence-sharded activations to the head split, with one
    all-to-all. xs: this rank's contiguous token share [t0, t1) (shard_slices
    over the L tokens) of every (b, h) slice, shape [n_slices, t1 - t0, ...].
    Returns this rank's slice share [s0, s1) (shard_slices over the slices)
    over all L tokens, shape [s1 - s0, L, ...] - the layout the head-split
    path runs on. Every stage of the method is independent per (b, h) slice,
    so this exchange (and heads_to_seq after it) is the only one a
    sequence-sharded caller needs."""
    import torch.distributed as dist
    inner = tuple(xs.shape[2:])
    shares = [shard_slices(1, n_slices, world, r) for r in range(world)]
    toks = [shard_slices(1, L, world, r) for r in range(world)]
    lr = toks[rank][1] - toks[rank][0]
    s0, s1 = shares[rank]
    n_me = s1 - s0
    assert xs.shape[0] == n_slices and xs.shape[1] == lr, (tuple(xs.shape), n_slices, lr)
    xb = _bytes_view(xs, 2)                     # [n_slices, lr, bytes per token]
    tb = xb.shape[2]
    # slices are the leading dim and go to ranks in order: the send buffer is xs itself
    send = xb.reshape(-1)
    recv = torch.empty(n_me * L * tb, dtype=torch.int8, device=xs.device)
    dist.all_to_all_single(recv, send,
                           output_split_sizes=[n_me * (b - a) * tb for a, b in toks],
                           input_split_sizes=[(b - a) * lr * tb for a, b in shares])
    out = torch.empty((n_me, L) + inner, dtype=xs.dtype, device=xs.device)
    ob, off = _bytes_view(out, 2), 0
    for a, b in toks:
        n = n_me * (b - a) * tb
        ob[:, a:b].copy_(recv[off:off + n].view(n_me, b - a, tb))
        off += n
    return out


def heads_to_seq(xh: torch.Tensor, n_slices: int, L: int, world: int, rank: int) -> torch.Tensor:
    """The inverse of seq_to_heads: this rank's slice share [s1 - s0, L, ...]
    back to its token share of every slice, [n_slices, t1 - t0, ...]."""
    import torch.distributed as dist
    inner = tuple(xh.shape[2:])
    shares = [shard_slices(1, n_slices, world, r) for r in range(world)]
    toks = [shard_slices(1, L, world, r) for r in range(world)]
    t0, t1 = toks[rank]
    s0, s1 = shares[rank]
    n_me = s1 - s0
    assert xh.shape[0] == n_me and xh.shape[1] == L, (tuple(xh.shape), n_me, L)
    xb = _bytes_view(xh, 2)                     # [n_me, L, bytes per token]
    tb = xb.shape[2]
    send = torch.cat([xb[:, a:b].reshape(-1) for a, b in toks])
    recv = torch.empty(n_slices * (t1 - t0) * tb, dtype=torch.int8, device=xh.device)
    dist.all_to_all_single(recv, send,
                           output_split_sizes=[(b - a) * (t1 - t0) * tb for a, b in shares],
                           input_split_sizes=[n_me * (b - a) * tb for a, b in toks])
    # sources send their slices in rank order, so the received bytes are the result
    out = torch.empty((n_slices, t1 - t0) + inner, dtype=xh.dtype, device=xh.device)
    _bytes_view(out, 2).view(-1).copy_(recv)
    return out
