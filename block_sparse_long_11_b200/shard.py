"""Sequence-sharded MoBA forward over several GPUs (one process per GPU).

The forward has no exchange step: every packed sequence is independent (its
blocks, gate and causal mask restart at its start, as the pages' block
partition does per sequence).  So a batch of sequences shards across ranks
as contiguous ranges of sequences -- zero-copy views of the packed
[T, H, d] tensors -- with no collective on the data path.  The only
collective is an optional all-gather of out / lse at the end, for callers
that want the whole result on every rank.

Ranges are balanced by the forward's work in closed form: a query at
position t of a sequence, in block j = t // B, attends t - jB + 1 keys of its
own block and min(topk - 1, j) full past blocks.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple


def sequence_work(L: int, block_size: int, topk: int) -> int:
    """Attended keys (per query head) of one sequence of L tokens."""
    B = block_size
    keys = 0
    for j in range((L + B - 1) // B):
        n = min(B, L - j * B)
        keys += n * (n + 1) // 2 + n * min(topk - 1, j) * B
    return keys


def plan_sequence_shards(seqlens: Sequence[int], world: int, block_size: int,
                         topk: int) -> List[Tuple[int, int]]:
    """Split sequences 0..n-1 into `world` contiguous ranges [a, b) with the
    largest range's work as small as possible (binary search on that bound,
    greedy fill).  Ranges may be empty when there are fewer sequences than
    ranks."""
    w = [sequence_work(int(L), block_size, topk) for L in seqlens]
    n = len(w)

    def fill(cap: int) -> Optional[List[Tuple[int, int]]]:
        out, a, acc = [], 0, 0
        for i, x in enumerate(w):
            if acc + x > cap and i > a:
                out.append((a, i))
                a, acc = i, 0
            acc += x
        out.append((a, n))
        return out if len(out) <= world else None

    lo, hi = max(w, default=0), sum(w)
    while lo < hi:
        mid = (lo + hi) // 2
        if fill(mid) is None:
            lo = mid + 1
        else:
            hi = mid
    ranges = fill(lo) or [(0, n)]
    while len(ranges) < world:
        ranges.append((n, n))
    return ranges


def moba_forward_sharded(q, k, v, seqlens: Sequence[int], block_size: int, topk: int,
                         softmax_scale: float = 0.0, rank: int = 0, world: int = 1,
                         gather: bool = False, group=None,
                         forward_fn: Optional[Callable] = None):
    """This rank's share of the forward of a packed batch.

    q, k, v: the whole packed batch (every rank holds it; only this rank's
    token range is read).  seqlens: host list of the sequence lengths.
    Returns (t0, t1, out_local, lse_local) for tokens [t0, t1) of the batch,
    or, with gather=True, (0, T, out, lse) of the whole batch on every rank
    (one all-gather over `group`).  forward_fn(q, k, v, cu_seqlens, block_size,
    topk, softmax_scale) -> (out, lse) defaults to the library's moba_forward.
    """
    import torch

    if forward_fn is None:
        from . import moba_forward as forward_fn
    ranges = plan_sequence_shards(seqlens, world, block_size, topk)
    cu = [0]
    for L in seqlens:
        cu.append(cu[-1] + int(L))
    a, b = ranges[rank]
    t0, t1 = cu[a], cu[b]
    if t1 > t0:
        cu_local = torch.tensor([c - t0 for c in cu[a:b + 1]], dtype=torch.int32,
                                device=q.device)
        out, lse = forward_fn(q[t0:t1], k[t0:t1], v[t0:t1], cu_local, block_size, topk,
                              softmax_scale)
    else:
        out = q.new_empty((0,) + tuple(q.shape[1:]))
        lse = torch.empty((0, q.shape[1]), dtype=torch.float32, device=q.device)
    if not gather or world == 1:
        return t0, t1, out, lse
    import torch.distributed as dist
    T = cu[-1]
    # pad every rank's piece to the longest range, gather, then cut
    span = max(cu[bb] - cu[aa] for aa, bb in ranges)
    o_pad = out.new_zeros((span,) + tuple(out.shape[1:]))
    l_pad = lse.new_zeros((span, lse.shape[1]))
    o_pad[:t1 - t0] = out
    l_pad[:t1 - t0] = lse
    o_all = [torch.empty_like(o_pad) for _ in range(world)]
    l_all = [torch.empty_like(l_pad) for _ in range(world)]
    dist.all_gather(o_all, o_pad, group=group)
    dist.all_gather(l_all, l_pad, group=group)
    out_full = out.new_empty((T,) + tuple(out.shape[1:]))
    lse_full = lse.new_empty((T, lse.shape[1]))
    for r, (aa, bb) in enumerate(ranges):
        n = cu[bb] - cu[aa]
        out_full[cu[aa]:cu[bb]] = o_all[r][:n]
        lse_full[cu[aa]:cu[bb]] = l_all[r][:n]
    return 0, T, out_full, lse_full
