"""Sequence sharding of the forward: the range planner (host logic, CPU) and
the sharded forward's rank logic with world size 2 over gloo on CPU (the
oracle stands in for each rank's forward)."""
import itertools
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synth
from block_sparse_long_11_b200 import shard
from oracle import moba_ref as R


@pytest.mark.parametrize("L,B,topk", [(1, 64, 3), (64, 64, 3), (1000, 64, 3), (4096, 512, 4),
                                      (5000, 256, 1), (777, 128, 100)])
def test_sequence_work_is_the_sum_of_attended_keys(L, B, topk):
    # the oracle counts a(t) row by row from the explicit definition
    assert shard.sequence_work(L, B, topk) == sum(R.attended_keys(t, B, topk) for t in range(L))


def _best_max(w, world):
    n = len(w)
    best = None
    for cuts in itertools.combinations(range(1, n), min(world, n) - 1):
        edges = (0,) + cuts + (n,)
        m = max(sum(w[a:b]) for a, b in zip(edges, edges[1:]))
        best = m if best is None else min(best, m)
    return best


@pytest.mark.parametrize("seqlens,world", [
    ([4096, 12288, 32768, 65536, 131072, 131072], 2),
    ([4096, 12288, 32768, 65536, 131072, 131072], 4),
    ([100, 200, 300, 400, 500], 3),
    ([5000], 4),
    ([7, 7, 7, 7], 8),
])
def test_plan_covers_in_order_and_is_optimal(seqlens, world):
    B, topk = 512, 4
    ranges = shard.plan_sequence_shards(seqlens, world, B, topk)
    assert len(ranges) == world
    edges = [a for a, _ in ranges] + [ranges[-1][1]]
    assert edges[0] == 0 and edges[-1] == len(seqlens)
    assert all(a <= b for a, b in ranges)
    assert all(ranges[i][1] == ranges[i + 1][0] for i in range(world - 1))
    w = [shard.sequence_work(L, B, topk) for L in seqlens]
    got = max(sum(w[a:b]) for a, b in ranges)
    assert got == _best_max(w, world)       # brute force over every contiguous split


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _oracle_forward(q, k, v, cu, B, topk, scale):
    res = R.forward(q.numpy(), k.numpy(), v.numpy(), cu.tolist(), q.shape[1], k.shape[1], B,
                    topk, scale=scale if scale > 0 else None)
    return torch.from_numpy(res["out"]), torch.from_numpy(res["lse"])


def _worker(rank, world, port, qout):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    w, x = synth.make_custom([70, 130, 45, 90], 2, 1, 8, 16, 3, seed=31)
    q, k, v = (x[n].float() for n in ("q", "k", "v"))
    t0, t1, out, lse = shard.moba_forward_sharded(q, k, v, w.seqlens, 16, 3, rank=rank,
                                                  world=world, gather=True,
                                                  forward_fn=_oracle_forward)
    dist.barrier()
    qout.put((rank, t0, t1, out.numpy(), lse.numpy()))
    dist.destroy_process_group()


def test_sharded_forward_world2_gathers_the_unsharded_result():
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, qq)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((qq.get(timeout=300) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w, x = synth.make_custom([70, 130, 45, 90], 2, 1, 8, 16, 3, seed=31)
    ref = R.forward(x["q"].float().numpy(), x["k"].float().numpy(), x["v"].float().numpy(),
                    w.cu_seqlens(), 2, 1, 16, 3)
    for rank, t0, t1, out, lse in res:
        assert (t0, t1) == (0, w.total_tokens)
        np.testing.assert_array_equal(out, ref["out"])
        np.testing.assert_array_equal(lse, ref["lse"])


# --- head-group sharding of one long sequence ----------------------------------------------
@pytest.mark.parametrize("Hq,Hkv,world", [(32, 8, 1), (32, 8, 2), (32, 8, 4), (32, 8, 8),
                                          (8, 2, 4), (8, 2, 8), (8, 2, 3), (16, 16, 3),
                                          (6, 3, 4), (4, 1, 4)])
def test_head_plan_covers_every_head_once_with_the_right_kv_heads(Hq, Hkv, world):
    G = Hq // Hkv
    plan = shard.plan_head_shards(Hq, Hkv, world)
    assert len(plan) == world
    covered = []
    for h0, h1, g0, g1 in plan:
        covered += list(range(h0, h1))
        if h1 == h0:
            continue
        # the library maps local query head i to local kv head i // (local Hq / local Hkv)
        assert (h1 - h0) % (g1 - g0) == 0
        Gl = (h1 - h0) // (g1 - g0)
        for h in range(h0, h1):
            assert g0 + (h - h0) // Gl == h // G
    assert covered == list(range(Hq))
    sizes = [h1 - h0 for h0, h1, _, _ in plan if h1 > h0]
    if world <= Hkv and Hkv % world == 0 or world % Hkv == 0 and G % (world // Hkv) == 0:
        assert len(set(sizes)) == 1 and len(sizes) == world   # perfectly even


def _head_worker(rank, world, port, qout):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    w, x = synth.make_custom([300], 4, 2, 8, 32, 3, seed=37)
    q, k, v = (x[n].float() for n in ("q", "k", "v"))
    h0, h1, out, lse = shard.moba_forward_head_sharded(q, k, v, x["cu_seqlens"], 32, 3, rank=rank,
                                                       world=world, gather=True,
                                                       forward_fn=_oracle_forward)
    dist.barrier()
    qout.put((rank, h0, h1, out.numpy(), lse.numpy()))
    dist.destroy_process_group()


def test_head_sharded_forward_world2_gathers_the_unsharded_result():
    ctx = mp.get_context("spawn")
    qq = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_head_worker, args=(r, 2, port, qq)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((qq.get(timeout=300) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w, x = synth.make_custom([300], 4, 2, 8, 32, 3, seed=37)
    ref = R.forward(x["q"].float().numpy(), x["k"].float().numpy(), x["v"].float().numpy(),
                    w.cu_seqlens(), 4, 2, 32, 3)
    for rank, h0, h1, out, lse in res:
        assert (h0, h1) == (0, 4)
        np.testing.assert_array_equal(out, ref["out"])
        np.testing.assert_array_equal(lse, ref["lse"])
