"""Sequence- and head-sharded MoBA forward over several GPUs (one process per GPU).

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

One long sequence (the 1M- and 10M-token workloads) shards by heads instead:
every query head routes on its own against the mean keys of its kv head and
attends only its kv head's keys, so a rank that holds a contiguous group of
kv heads and their query heads -- the layout a tensor-parallel attention
layer produces anyway -- runs the ordinary forward on its local [T, H/N, d]
tensors, again with no exchange step (an optional all-gather of out / lse
along the heads at the end).
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


def plan_head_shards(n_heads: int, n_kv_heads: int, world: int) -> List[Tuple[int, int, int, int]]:
    """(h0, h1, g0, g1) for every rank: query heads [h0, h1) and the kv heads
    [g0, g1) they read.  Every query head costs the same (same sequences, same
    selection sizes), so the query heads are split evenly, in order:
      * world <= n_kv_heads: whole groups -- the kv heads split as evenly as
        possible, each with its G = n_heads / n_kv_heads query heads;
      * world a multiple of n_kv_heads and G a multiple of world / n_kv_heads:
        each group's query heads split across world / n_kv_heads ranks, which
        each hold a copy of that group's kv head;
      * otherwise whole groups again, with the ranks beyond n_kv_heads idle.
    A rank's query heads then map to its kv heads exactly as in the library
    (local query head i reads local kv head i / (local query heads / local kv
    heads))."""
    if n_heads % n_kv_heads != 0 or world < 1:
        raise ValueError("n_heads must be a multiple of n_kv_heads and world >= 1")
    G = n_heads // n_kv_heads
    R = world // n_kv_heads
    out = []
    if world > n_kv_heads and world % n_kv_heads == 0 and G % R == 0:
        per = G // R
        for r in range(world):
            g, part = divmod(r, R)
            out.append((g * G + part * per, g * G + (part + 1) * per, g, g + 1))
        return out
    for r in range(world):
        g0 = (r * n_kv_heads) // world if world <= n_kv_heads else min(r, n_kv_heads)
        g1 = ((r + 1) * n_kv_heads) // world if world <= n_kv_heads else min(r + 1, n_kv_heads)
        out.append((g0 * G, g1 * G, g0, g1))
    return out


def moba_forward_head_sharded(q, k, v, cu_seqlens, block_size: int, topk: int,
                              softmax_scale: float = 0.0, rank: int = 0, world: int = 1,
                              gather: bool = False, group=None,
                              forward_fn: Optional[Callable] = None):
    """This rank's heads of the forward, from the whole q [T, Hq, d] and k, v
    [T, Hkv, d]: the rank's head slices (plan_head_shards) are copied out
    contiguous and run through the ordinary forward.  (A rank whose tensors
    already hold only its heads calls moba_forward on them directly: that is
    the same computation.)
    Returns (h0, h1, out_local [T, h1 - h0, d], lse_local [T, h1 - h0]), or
    with gather=True (0, Hq, out, lse) of every head on every rank (one
    all-gather over `group`).  forward_fn as in moba_forward_sharded.
    """
    import torch

    if forward_fn is None:
        from . import moba_forward as forward_fn
    Hq, Hkv = q.shape[1], k.shape[1]
    h0, h1, g0, g1 = plan_head_shards(Hq, Hkv, world)[rank]
    if h1 > h0:
        ql = q[:, h0:h1].contiguous()
        kl = k[:, g0:g1].contiguous()
        vl = v[:, g0:g1].contiguous()
        out, lse = forward_fn(ql, kl, vl, cu_seqlens, block_size, topk, softmax_scale)
    else:
        out = q.new_empty((q.shape[0], 0, q.shape[2]))
        lse = torch.empty((q.shape[0], 0), dtype=torch.float32, device=q.device)
    if not gather or world == 1:
        return h0, h1, out, lse
    import torch.distributed as dist
    plan = plan_head_shards(Hq, Hkv, world)
    span = max(b - a for a, b, _, _ in plan)
    T, d = q.shape[0], q.shape[2]
    o_pad = out.new_zeros((T, span, d))
    l_pad = lse.new_zeros((T, span))
    o_pad[:, :h1 - h0] = out
    l_pad[:, :h1 - h0] = lse
    o_all = [torch.empty_like(o_pad) for _ in range(world)]
    l_all = [torch.empty_like(l_pad) for _ in range(world)]
    dist.all_gather(o_all, o_pad, group=group)
    dist.all_gather(l_all, l_pad, group=group)
    out_full = out.new_empty((T, Hq, d))
    lse_full = lse.new_empty((T, Hq))
    for r, (a, b, _, _) in enumerate(plan):
        out_full[:, a:b] = o_all[r][:, :b - a]
        lse_full[:, a:b] = l_all[r][:, :b - a]
    return 0, Hq, out_full, lse_full
