"""Seeded synthetic inputs for the MoBA causal prefill forward.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no pooling, scoring, selection or attention).  Both the
CUDA path and the CPU oracle are fed from here, so a parity test hands the
same bf16 bits to both sides.

Layout of every tensor it returns (packed variable-length "THD" layout):

  q  bf16 [T, Hq,  d]     k, v  bf16 [T, Hkv, d]     cu_seqlens int32 [n_seqs + 1]

Values are drawn in fp32 from a seeded ``torch.Generator`` on the requested
device and rounded to bf16.  Large tensors are drawn in fixed chunks of
``CHUNK_TOKENS`` tokens, each chunk seeded from (seed, tensor, chunk index), so
the bits do not depend on available memory.  CPU and CUDA generators give
different streams for the same seed; a test draws once and feeds both sides.

Workload shapes follow the pages' settings: the scaling-law shape of the
experiments section, the Llama-8B-1M setting (block 4096, top-k 12, 32 query
heads over 8 KV heads, head dim 128) of the "大語言模型評估" section, and
lengths up to 10M tokens from the "效率和可擴展性" section of the MoBA
write-up "同一天，DeepSeek和月之暗面發表了關于改進注意力機制的論文".
The real corpora, RULER and needle-in-a-haystack sets are not used: the
planted-needle workload below is a synthetic stand-in.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch

CHUNK_TOKENS = 65536


@dataclasses.dataclass
class Workload:
    name: str
    seqlens: list
    n_heads: int
    n_kv_heads: int
    head_dim: int
    block_size: int
    topk: int
    seed: int
    kind: str = "normal"          # "normal" | "needle" | "head_scaled"

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens))

    @property
    def n_seqs(self) -> int:
        return len(self.seqlens)

    def cu_seqlens(self) -> list:
        cu = [0]
        for L in self.seqlens:
            cu.append(cu[-1] + int(L))
        return cu


# The five workloads of the benchmark table, named by what they are.
WORKLOADS = {
    "single_2k_d64_b256": Workload("single_2k_d64_b256", [2048], 1, 1, 64, 256, 3, 1001),
    "scaling_4x8k_h16_b512": Workload("scaling_4x8k_h16_b512", [8192] * 4, 16, 16, 128, 512, 3, 1002),
    "needle_2x32k_h16_b512": Workload("needle_2x32k_h16_b512", [32768] * 2, 16, 16, 128, 512, 3, 1003,
                                      kind="needle"),
    "varlen_377k_gqa32x8_b4096": Workload("varlen_377k_gqa32x8_b4096",
                                          [4096, 12288, 32768, 65536, 131072, 131072], 32, 8, 128,
                                          4096, 12, 1004, kind="head_scaled"),
    "long_1m_gqa32x8_b4096": Workload("long_1m_gqa32x8_b4096", [1048576], 32, 8, 128, 4096, 12, 1005),
    "long_10m_gqa8x2_b4096": Workload("long_10m_gqa8x2_b4096", [10485760], 8, 2, 128, 4096, 12, 1006),
}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return g


def _sub_seed(seed: int, tensor_id: int, chunk: int) -> int:
    # Plain integer mixing so each (tensor, chunk) has its own stream.
    return (seed * 1_000_003 + tensor_id * 7_919 + chunk * 104_729 + 12_345) % (2 ** 61 - 1)


def normal_bf16(shape: Sequence[int], seed: int, tensor_id: int, device="cpu", std: float = 1.0):
    """bf16 tensor of iid N(0, std^2) values, drawn chunk by chunk along dim 0."""
    shape = tuple(int(s) for s in shape)
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    rows = shape[0]
    per_row = 1
    for s in shape[1:]:
        per_row *= s
    r = 0
    chunk = 0
    while r < rows:
        n = min(CHUNK_TOKENS, rows - r)
        g = _gen(device, _sub_seed(seed, tensor_id, chunk))
        x = torch.randn((n,) + shape[1:], generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        out[r:r + n].copy_(x)
        del x
        r += n
        chunk += 1
    return out


def make_inputs(w: Workload, device="cpu"):
    """Draw q, k, v and cu_seqlens for workload ``w`` on ``device``.

    Returns a dict with q, k, v (bf16), cu_seqlens (int32, same device) and
    ``meta`` (plain Python description of what was planted, for needle runs).
    """
    T = w.total_tokens
    q = normal_bf16((T, w.n_heads, w.head_dim), w.seed, 1, device)
    k = normal_bf16((T, w.n_kv_heads, w.head_dim), w.seed, 2, device)
    v = normal_bf16((T, w.n_kv_heads, w.head_dim), w.seed, 3, device)
    meta = {}
    if w.kind == "head_scaled":
        # per-head scale drawn U(0.5, 2) separately for q, k and v
        g = _gen("cpu", _sub_seed(w.seed, 10, 0))
        sq = 0.5 + 1.5 * torch.rand(w.n_heads, generator=g, dtype=torch.float32)
        sk = 0.5 + 1.5 * torch.rand(w.n_kv_heads, generator=g, dtype=torch.float32)
        sv = 0.5 + 1.5 * torch.rand(w.n_kv_heads, generator=g, dtype=torch.float32)
        for t, s in ((q, sq), (k, sk), (v, sv)):
            s_dev = s.to(device)
            r = 0
            while r < T:
                n = min(CHUNK_TOKENS, T - r)
                t[r:r + n].copy_((t[r:r + n].float() * s_dev[None, :, None]))
                r += n
        meta["head_scales"] = {"q": sq.tolist(), "k": sk.tolist(), "v": sv.tolist()}
    elif w.kind == "needle":
        meta["needles"] = plant_needles(q, k, w, device)
    cu = torch.tensor(w.cu_seqlens(), dtype=torch.int32, device=device)
    return {"q": q, "k": k, "v": v, "cu_seqlens": cu, "meta": meta}


def plant_needles(q, k, w: Workload, device):
    """Plant one needle block per (sequence, kv head) and route 1% of queries to it.

    The needle block index n is drawn uniformly from [1, nb/2 - 1] (first half,
    never block 0).  Its keys become 3*u + N(0, 0.5^2), with u a seeded unit
    vector per head.  1% of the query positions in blocks after n (seeded) get
    q = N(0, 1) + 3*u.  Requires n_heads == n_kv_heads (the needle workload has
    16 heads over 16 KV heads).
    """
    assert w.n_heads == w.n_kv_heads
    g = _gen("cpu", _sub_seed(w.seed, 20, 0))
    d, B = w.head_dim, w.block_size
    u = torch.randn(w.n_kv_heads, d, generator=g, dtype=torch.float32)
    u = u / u.norm(dim=1, keepdim=True)
    cu = w.cu_seqlens()
    needles = []
    for s, L in enumerate(w.seqlens):
        nb = L // B
        for h in range(w.n_kv_heads):
            n = int(torch.randint(1, max(2, nb // 2), (1,), generator=g).item())
            start = cu[s] + n * B
            noise = 0.5 * torch.randn(B, d, generator=g, dtype=torch.float32)
            k[start:start + B, h, :] = (3.0 * u[h][None, :] + noise).to(device=device, dtype=k.dtype)
            first = (n + 1) * B
            cand = L - first
            m = max(1, cand // 100)
            pos = torch.randperm(cand, generator=g)[:m] + first
            pos, _ = torch.sort(pos)
            z = torch.randn(m, d, generator=g, dtype=torch.float32)
            rows = cu[s] + pos
            q[rows.to(device), h, :] = (z + 3.0 * u[h][None, :]).to(device=device, dtype=q.dtype)
            needles.append({"seq": s, "head": h, "block": n, "positions": pos.tolist()})
    return needles


def make_custom(seqlens, n_heads, n_kv_heads, head_dim, block_size, topk, seed, device="cpu",
                kind="normal"):
    """Inputs for an ad-hoc shape (parity cases: ragged tails, tiny shapes)."""
    w = Workload("custom", list(seqlens), n_heads, n_kv_heads, head_dim, block_size, topk, seed, kind)
    return w, make_inputs(w, device)


def make_decode(n_seqs, max_len, n_heads, n_kv_heads, head_dim, seed, device="cpu"):
    """Padded KV caches [n_seqs, max_len, Hkv, d] and one query per sequence
    [n_seqs, Hq, d] (bf16, iid N(0, 1)) for decode steps.  Cache positions a
    sequence does not use yet hold values too; they must never be read."""
    q = normal_bf16((n_seqs, n_heads, head_dim), seed, 40, device)
    kc = torch.empty((n_seqs, max_len, n_kv_heads, head_dim), dtype=torch.bfloat16, device=device)
    vc = torch.empty_like(kc)
    for s in range(n_seqs):
        kc[s].copy_(normal_bf16((max_len, n_kv_heads, head_dim), seed, 41 + 2 * s, device))
        vc[s].copy_(normal_bf16((max_len, n_kv_heads, head_dim), seed, 42 + 2 * s, device))
    return {"q": q, "k_cache": kc, "v_cache": vc}


def sample_rows(w: Workload, n_rows: int, seed: int):
    """Seeded, stratified sample of (token, head) rows for full-size parity.

    Always includes, for every sequence, a row in its block 0 and one in its
    last block; the rest are uniform over all T * Hq rows.  Returns a sorted
    list of (t_global, h) pairs without repeats.
    """
    g = _gen("cpu", _sub_seed(seed, 30, 0))
    cu = w.cu_seqlens()
    picks = set()
    for s, L in enumerate(w.seqlens):
        B = w.block_size
        nb = (L + B - 1) // B
        for blk in (0, nb - 1):
            lo = cu[s] + blk * B
            hi = min(cu[s] + L, lo + B)
            t = lo + int(torch.randint(0, hi - lo, (1,), generator=g).item())
            h = int(torch.randint(0, w.n_heads, (1,), generator=g).item())
            picks.add((t, h))
    total = w.total_tokens * w.n_heads
    while len(picks) < n_rows:
        r = int(torch.randint(0, total, (1,), generator=g).item())
        picks.add((r // w.n_heads, r % w.n_heads))
    return sorted(picks)


def sample_keys(w: Workload, n_keys: int, seed: int):
    """Seeded, stratified sample of (token, kv head) keys, as sample_rows:
    for every sequence a key in its block 0 (the block most rows route to)
    and one in its last block, the rest uniform over all T * Hkv keys.
    Returns a sorted list of (t_global, g) pairs without repeats."""
    g = _gen("cpu", _sub_seed(seed, 31, 0))
    cu = w.cu_seqlens()
    picks = set()
    for s, L in enumerate(w.seqlens):
        B = w.block_size
        nb = (L + B - 1) // B
        for blk in (0, nb - 1):
            lo = cu[s] + blk * B
            hi = min(cu[s] + L, lo + B)
            t = lo + int(torch.randint(0, hi - lo, (1,), generator=g).item())
            kv = int(torch.randint(0, w.n_kv_heads, (1,), generator=g).item())
            picks.add((t, kv))
    total = w.total_tokens * w.n_kv_heads
    while len(picks) < n_keys:
        r = int(torch.randint(0, total, (1,), generator=g).item())
        picks.add((r // w.n_kv_heads, r % w.n_kv_heads))
    return sorted(picks)
