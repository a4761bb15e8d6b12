"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Small shapes are compared row by row over every (token, head); the benchmark
workloads at full size are compared on seeded, stratified samples of rows in
the same launch configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

import block_sparse_long_11_b200 as mb
import synth
from oracle import moba_ref as R
from tests import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_long_11_b200 import build
    build.build()
    assert torch.cuda.is_available()
    mb.lib()


def _run(w, x, chunk=None, ws=None):
    out, lse, idx = mb.moba_forward(x["q"], x["k"], x["v"], x["cu_seqlens"], w.block_size, w.topk,
                                    chunk_tokens=chunk, workspace=ws, return_idx=True)
    mb.moba_check(ws)
    torch.cuda.synchronize()
    return out, lse, idx


# --- gate alone -----------------------------------------------------------------
@pytest.mark.parametrize("topk", [3, 8])
def test_gate_single_2k_d64(topk):
    w = synth.WORKLOADS["single_2k_d64_b256"]
    x = synth.make_inputs(w, DEV)
    idx = mb.moba_gate(x["q"], x["k"], x["cu_seqlens"], w.block_size, topk)
    mb.moba_check()
    ref = R.forward(P.bits(x["q"]), P.bits(x["k"]), P.bits(x["v"]), np.array(w.cu_seqlens()),
                    1, 1, w.block_size, topk)
    g = idx.cpu().numpy()
    qb, kb = P.bits(x["q"]), P.bits(x["k"])
    kbar = R.block_means(kb, w.block_size)
    exact = (g == ref["idx"]).all(axis=-1)
    assert (exact | ref["tie"]).all(), np.argwhere(~(exact | ref["tie"]))[:5]
    for t, h in np.argwhere(ref["tie"] & ~exact):
        j = t // w.block_size
        got = [int(v) for v in g[t, h] if v >= 0]
        assert P.valid_selection(R.gate_scores(qb[t, h], kbar[:, 0, :], j), j, topk, got)


# (d, B, top-k): the tcgen05 gate (top-k <= 16; more than 256 past blocks
# recompute the scores for a second, bounded pass) and the CUDA-core gate (17-64)
GATE_LONG = [(64, 64, 5), (128, 128, 5), (128, 128, 12), (64, 64, 20), (128, 128, 40)]


@pytest.mark.parametrize("d,B,topk", GATE_LONG, ids=[f"d{c[0]}_b{c[1]}_k{c[2]}" for c in GATE_LONG])
def test_gate_more_than_256_past_blocks(d, B, topk):
    """Rows with up to ~320 past blocks.  Kv head 0 also holds five bit-identical
    copies of one block (keys 3u + N(0,1), u a unit vector), so its rows see
    exact score ties, often straddling the cut: a selected copy implies every
    lower-index copy is selected too (the lower index wins a tie)."""
    L = B * 322 + 37
    w, x = synth.make_custom([L], 4, 2, d, B, topk, seed=31 + d + topk, device=DEV)
    copies = [3, 40, 130, 260, 300]
    gen = torch.Generator(device="cpu").manual_seed(5 + d)
    u = torch.randn(d, generator=gen)
    u /= u.norm()
    blk = 3.0 * u[None, :] + torch.randn(B, d, generator=gen)
    for c in copies:
        x["k"][c * B:(c + 1) * B, 0, :] = blk.to(device=DEV, dtype=torch.bfloat16)
    idx = mb.moba_gate(x["q"], x["k"], x["cu_seqlens"], B, topk)
    mb.moba_check()
    g = idx.cpu().numpy()
    qb, kb = P.bits(x["q"]), P.bits(x["k"])
    kbar = R.block_means(kb, B)
    assert all(np.array_equal(kbar[c, 0], kbar[3, 0]) for c in copies)
    rows = list(range(0, L, 97)) + [L - 1, B * 257, B * 300 + 5] + list(range(B * 301, L, 11))
    straddle = 0
    for t in rows:
        for h in range(4):
            j = t // B
            sc = R.gate_scores(qb[t, h], kbar[:, h // 2, :], j)
            sel, tie = R.select_blocks(sc, j, topk)
            got = [int(v) for v in g[t, h] if v >= 0]
            assert got == sel or (tie and P.valid_selection(sc, j, topk, got)), (t, h, got, sel)
            if h < 2 and j > copies[-1]:
                inside = [c for c in copies if c in got]
                assert inside == copies[:len(inside)], (t, h, got)
                straddle += 0 < len(inside) < len(copies)
    if topk - 1 < len(copies):   # the copies straddle the cut on many rows
        assert straddle > 20, straddle


# --- whole forward, every row ----------------------------------------------------
@pytest.mark.parametrize("topk", [3, 8])
def test_forward_single_2k_d64_all_rows(topk):
    w = synth.WORKLOADS["single_2k_d64_b256"]
    w = synth.Workload(w.name, w.seqlens, 1, 1, 64, 256, topk, w.seed)
    x = synth.make_inputs(w, DEV)
    out, lse, idx = _run(w, x)
    st = P.check_rows(x, w, out, lse, idx, P.all_rows(w))
    if topk == 8:   # top-k >= number of blocks: full causal attention
        qf = x["q"].float().permute(1, 0, 2)[None]
        kf = x["k"].float().permute(1, 0, 2)[None]
        vf = x["v"].float().permute(1, 0, 2)[None]
        full = torch.nn.functional.scaled_dot_product_attention(qf, kf, vf, is_causal=True)
        d = (full[0].permute(1, 0, 2) - out.float()).abs()
        assert d.max().item() <= P.OUT_MAX_ABS and d.mean().item() <= P.OUT_MEAN_ABS
    assert st["rows"] == 2048


SMALL = [
    # seqlens, Hq, Hkv, d, B, topk, chunk
    ([1000, 3000, 129, 2125], 8, 2, 128, 128, 4, None),   # ragged varlen, GQA, d128
    ([777, 1280, 64], 4, 4, 64, 64, 3, None),              # d64, B=64
    ([4096], 2, 1, 128, 256, 1, None),                    # top-1: own block only
    ([2048, 1500], 4, 2, 128, 256, 16, None),             # top-k >= number of blocks
    ([5000, 1234], 4, 1, 128, 128, 5, 777),               # several query passes, odd chunk
    ([50, 63, 1], 2, 2, 64, 64, 3, None),                 # no full block at all
    ([3333], 6, 3, 64, 192, 2, 1000),                     # B = 192, odd chunk
]


@pytest.mark.parametrize("case", SMALL, ids=[str(i) for i in range(len(SMALL))])
def test_forward_small_all_rows(case):
    seqlens, Hq, Hkv, d, B, topk, chunk = case
    w, x = synth.make_custom(seqlens, Hq, Hkv, d, B, topk, seed=700 + len(seqlens), device=DEV)
    out, lse, idx = _run(w, x, chunk=chunk)
    P.check_rows(x, w, out, lse, idx, P.all_rows(w))


def test_forward_running_max_moves_often():
    """Keys whose norm ramps up along every block push each row's max up tile
    after tile, so the softmax keeps moving its running max and rescaling O."""
    w, x = synth.make_custom([6144, 2500], 4, 2, 128, 1024, 3, seed=907, device=DEV)
    T = w.total_tokens
    ramp = 1.0 + 5.0 * (torch.arange(T, device=DEV) % 1024).float() / 1024.0
    x["k"].copy_((x["k"].float() * ramp[:, None, None]).to(torch.bfloat16))
    x["q"].mul_(3.0)
    out, lse, idx = _run(w, x)
    # Attention here is nearly one-hot with |o| up to ~4, so rounding P and the
    # output to bf16 (unit roundoff 2^-8 each) costs up to ~2^-7 |o| by itself:
    # the budget is 1e-2 + 2^-7 |o|.  A wrong rescale would be off by O(|o|).
    P.check_rows(x, w, out, lse, idx, P.all_rows(w), out_rtol=2.0 ** -7)


def test_forward_topk_above_16_and_explicit_scale():
    """top-k 20 (the CUDA-core gate path) and a caller-given softmax scale."""
    w, x = synth.make_custom([6000, 1111], 4, 2, 128, 128, 20, seed=911, device=DEV)
    out, lse, idx = mb.moba_forward(x["q"], x["k"], x["v"], x["cu_seqlens"], 128, 20,
                                    softmax_scale=0.05, return_idx=True)
    mb.moba_check()
    torch.cuda.synchronize()
    P.check_rows(x, w, out, lse, idx, P.all_rows(w), scale=0.05)


def test_forward_deterministic_and_chunk_invariant():
    w, x = synth.make_custom([3000, 2000], 8, 2, 128, 128, 4, seed=901, device=DEV)
    a = _run(w, x)
    b = _run(w, x)
    c = _run(w, x, chunk=1111)
    for u, v in zip(a, b):
        assert torch.equal(u, v)
    for u, v in zip(a, c):
        assert torch.equal(u, v)


def test_forward_empty_and_bad_seqlens():
    w, x = synth.make_custom([256], 2, 2, 64, 64, 3, seed=5, device=DEV)
    e = torch.empty((0, 2, 64), dtype=torch.bfloat16, device=DEV)
    cu0 = torch.zeros(2, dtype=torch.int32, device=DEV)
    out, lse = mb.moba_forward(e, e, e, cu0, 64, 3)
    assert out.shape == (0, 2, 64)
    bad = torch.tensor([0, 200, 100, 256], dtype=torch.int32, device=DEV)   # not monotone
    ws = mb.Workspace()
    mb.moba_forward(x["q"], x["k"], x["v"], bad, 64, 3, workspace=ws)
    with pytest.raises(mb.MobaError) as ei:
        mb.moba_check(ws)
    assert ei.value.code == 6
    # the same workspace runs clean afterwards
    out, lse = mb.moba_forward(x["q"], x["k"], x["v"], x["cu_seqlens"], 64, 3, workspace=ws)
    mb.moba_check(ws)


# --- dense causal attention through the same kernel (the full <-> sparse switch) -------
FULL = [
    # seqlens, Hq, Hkv, d
    ([1500, 700, 2100], 4, 2, 128),     # ragged varlen, GQA
    ([777, 1280, 64, 1], 4, 4, 64),     # d64, a one-token sequence
    ([3000], 2, 1, 128),                # one sequence, 12 units of 256 rows per head
]


@pytest.mark.parametrize("case", FULL, ids=[str(i) for i in range(len(FULL))])
def test_forward_full_all_rows(case):
    seqlens, Hq, Hkv, d = case
    w, x = synth.make_custom(seqlens, Hq, Hkv, d, 256, 1, seed=950 + len(seqlens), device=DEV)
    out, lse = mb.moba_forward_full(x["q"], x["k"], x["v"], x["cu_seqlens"])
    mb.moba_check()
    torch.cuda.synchronize()
    P.check_full_rows(x, w, out, lse, P.all_rows(w))


def test_forward_full_matches_topk_covering_every_block():
    """moba_forward with top-k >= blocks per sequence is full causal attention
    too: both paths agree with each other within the output tolerance."""
    w, x = synth.make_custom([2048, 1111], 4, 2, 128, 128, 16, seed=961, device=DEV)
    full, lse_f = mb.moba_forward_full(x["q"], x["k"], x["v"], x["cu_seqlens"], softmax_scale=0.07)
    sparse, lse_s = mb.moba_forward(x["q"], x["k"], x["v"], x["cu_seqlens"], 128, 16,
                                    softmax_scale=0.07)
    mb.moba_check()
    torch.cuda.synchronize()
    d = (full.float() - sparse.float()).abs()
    assert d.max().item() <= P.OUT_MAX_ABS and d.mean().item() <= P.OUT_MEAN_ABS
    assert (lse_f - lse_s).abs().max().item() <= P.LSE_MAX_ABS
    P.check_full_rows(x, w, full, lse_f, P.all_rows(w)[::7], scale=0.07)


def test_forward_full_2x32k_sampled():
    """Units of up to 256 K/V steps, longest first."""
    w, x = synth.make_custom([32768, 20000], 16, 4, 128, 256, 1, seed=963, device=DEV)
    out, lse = mb.moba_forward_full(x["q"], x["k"], x["v"], x["cu_seqlens"])
    mb.moba_check()
    torch.cuda.synchronize()
    rows = synth.sample_rows(w, 256, 17)
    P.check_full_rows(x, w, out, lse, rows)


# --- backward (selection of the forward held fixed) ----------------------------------------
BWD = [
    # seqlens, Hq, Hkv, d, B, topk
    ([700, 1300], 4, 2, 128, 128, 4),     # ragged varlen, GQA, gate active
    ([900], 2, 2, 64, 64, 3),             # d64
    ([1024, 333], 4, 1, 128, 256, 16),    # top-k covers every block: full causal
]


def _oracle_saved_inputs(w, x, seed):
    """The backward's saved inputs from the ORACLE forward: out rounded to
    bf16 and lse to fp32 (the precisions the forward stores), its selection,
    and a synthetic dout."""
    cu = w.cu_seqlens()
    fw = R.forward(P.bits(x["q"]), P.bits(x["k"]), P.bits(x["v"]), cu, w.n_heads, w.n_kv_heads,
                   w.block_size, w.topk)
    out = torch.from_numpy(fw["out"]).to(torch.bfloat16)
    lse = torch.from_numpy(fw["lse"]).to(torch.float32)
    idx = torch.from_numpy(fw["idx"]).to(torch.int32)
    dout = synth.normal_bf16(tuple(x["q"].shape), seed, 50, DEV)
    return out.to(DEV), lse.to(DEV), idx.to(DEV), dout


def _check_backward(w, x, out, lse, idx, dout, dq, dk, dv):
    """GPU gradients against the oracle's saved-statistics backward on the same
    inputs.  Tolerance per element: 2^-7 of the oracle's sum of the absolute
    values of the element's terms, plus 1e-4 of the largest such sum.  The
    kernels round P (for dV) and dS (for dK, dQ) once each to bf16 before their
    MMAs -- unit roundoff 2^-8, so at most 2^-8 of the absolute-term sum --
    with fp32 products and sums otherwise; the bound allows twice that."""
    ref = R.backward_saved(P.bits(x["q"]), P.bits(x["k"]), P.bits(x["v"]), w.cu_seqlens(),
                           R.as_f64(P.bits(dout)), R.as_f64(P.bits(out)),
                           lse.double().cpu().numpy(), idx.cpu().numpy(), w.n_heads,
                           w.n_kv_heads, w.block_size, w.topk)
    worst = {}
    for name, got in (("dq", dq), ("dk", dk), ("dv", dv)):
        g = got.double().cpu().numpy()
        r, a = ref[name], ref[name + "_abs"]
        err = np.abs(g - r)
        budget = 2.0 ** -7 * a + 1e-4 * a.max()
        assert np.all(err <= budget), (name, float((err / budget).max()))
        worst[name] = float((err / np.maximum(a, 1e-30)).max())
    return worst


@pytest.mark.parametrize("case", BWD, ids=[str(i) for i in range(len(BWD))])
def test_backward_matches_oracle_on_saved_statistics(case):
    """dq, dk, dv (tensor cores) against the oracle backward, both fed the
    oracle forward's out / lse / selection: a tight elementwise check."""
    seqlens, Hq, Hkv, d, B, topk = case
    w, x = synth.make_custom(seqlens, Hq, Hkv, d, B, topk, seed=930 + len(seqlens), device=DEV)
    out, lse, idx, dout = _oracle_saved_inputs(w, x, 930 + len(seqlens))
    dq, dk, dv = mb.moba_backward(x["q"], x["k"], x["v"], out, lse, dout, x["cu_seqlens"], idx,
                                  B, topk)
    mb.moba_check()
    torch.cuda.synchronize()
    _check_backward(w, x, out, lse, idx, dout, dq, dk, dv)


def test_backward_after_the_gpu_forward():
    """The whole path: the GPU forward's out / lse / selection into the GPU
    backward, against the oracle's exact backward on that selection (its D
    uses the exact fp64 output, so the bf16 rounding and the forward's own
    error in out enter here: 1e-2 relative in norm, 5e-2 of the largest
    magnitude per element)."""
    seqlens, Hq, Hkv, d, B, topk = BWD[0]
    w, x = synth.make_custom(seqlens, Hq, Hkv, d, B, topk, seed=931, device=DEV)
    T = w.total_tokens
    dout = synth.normal_bf16((T, Hq, d), 931, 50, DEV)
    out, lse, idx = mb.moba_forward(x["q"], x["k"], x["v"], x["cu_seqlens"], B, topk,
                                    return_idx=True)
    dq, dk, dv = mb.moba_backward(x["q"], x["k"], x["v"], out, lse, dout, x["cu_seqlens"], idx,
                                  B, topk)
    mb.moba_check()
    torch.cuda.synchronize()
    ref = R.backward(P.bits(x["q"]), P.bits(x["k"]), P.bits(x["v"]), w.cu_seqlens(),
                     R.as_f64(P.bits(dout)), Hq, Hkv, B, topk, idx=idx.cpu().numpy())
    for name, got in (("dq", dq), ("dk", dk), ("dv", dv)):
        g = got.double().cpu().numpy()
        r = ref[name]
        rel = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
        assert rel <= 1e-2, (name, rel)
        assert np.abs(g - r).max() <= 5e-2 * max(1.0, np.abs(r).max()), name


def test_backward_deterministic_and_chunk_invariant():
    """dq sums each row's per-block partials in block order, and dk, dv sum a
    bucket's rows in ascending (token, head) order (the stable fill): all
    three identical from run to run and for any query chunking of the dq
    partial slots."""
    w, x = synth.make_custom([3000, 2000], 8, 2, 128, 256, 5, seed=935, device=DEV)
    out, lse, idx, dout = _oracle_saved_inputs(w, x, 935)
    args = (x["q"], x["k"], x["v"], out, lse, dout, x["cu_seqlens"], idx, 256, 5)
    a = mb.moba_backward(*args)
    b = mb.moba_backward(*args)
    c = mb.moba_backward(*args, chunk_tokens=1111)
    mb.moba_check()
    torch.cuda.synchronize()
    for i in range(3):
        assert torch.equal(a[i], b[i]) and torch.equal(a[i], c[i]), i


def test_backward_varlen_377k_gqa32x8_b4096_sampled():
    """The backward at a benchmark workload's full size (377K tokens, six
    sequences of 4K to 128K, 32 q / 8 kv heads, block 4096, top-k 12) after
    the GPU forward: dq of 512 sampled rows and dk, dv of 48 sampled keys
    against the oracle's sampled saved-statistics backward on the same out,
    lse and selection, elementwise with the budget of _check_backward (its
    largest-sum term taken over the sample)."""
    w = synth.WORKLOADS["varlen_377k_gqa32x8_b4096"]
    x = synth.make_inputs(w, DEV)
    out, lse, idx = _run(w, x)
    dout = synth.normal_bf16(tuple(x["q"].shape), w.seed, 50, DEV)
    dq, dk, dv = mb.moba_backward(x["q"], x["k"], x["v"], out, lse, dout, x["cu_seqlens"], idx,
                                  w.block_size, w.topk)
    mb.moba_check()
    torch.cuda.synchronize()
    rows = synth.sample_rows(w, 512, 21)
    keys = synth.sample_keys(w, 48, 22)
    ref = R.backward_saved_sample(P.bits(x["q"]), P.bits(x["k"]), P.bits(x["v"]), w.cu_seqlens(),
                                  P.bits(dout), P.bits(out), lse.double().cpu().numpy(),
                                  idx.cpu().numpy(), w.n_heads, w.n_kv_heads, w.block_size,
                                  w.topk, rows=rows, keys=keys)
    rt = torch.tensor(rows, device=DEV)
    kt = torch.tensor(keys, device=DEV)
    got = {"dq": dq[rt[:, 0], rt[:, 1]], "dk": dk[kt[:, 0], kt[:, 1]],
           "dv": dv[kt[:, 0], kt[:, 1]]}
    for name, g in got.items():
        g = g.double().cpu().numpy()
        r, a = ref[name], ref[name + "_abs"]
        budget = 2.0 ** -7 * a + 1e-4 * a.max()
        assert np.all(np.abs(g - r) <= budget), (name, float((np.abs(g - r) / budget).max()))


def test_backward_rejects_a_malformed_selection():
    w, x = synth.make_custom([1000], 2, 2, 64, 64, 3, seed=936, device=DEV)
    out, lse, idx, dout = _oracle_saved_inputs(w, x, 936)
    bad = idx.clone()
    bad[500, 1, 0] = 14   # beyond the row's own block (j = 7)
    ws = mb.Workspace()
    mb.moba_backward(x["q"], x["k"], x["v"], out, lse, dout, x["cu_seqlens"], bad, 64, 3,
                     workspace=ws)
    with pytest.raises(mb.MobaError) as ei:
        mb.moba_check(ws)
    assert ei.value.code == 7
    mb.moba_backward(x["q"], x["k"], x["v"], out, lse, dout, x["cu_seqlens"], idx, 64, 3,
                     workspace=ws)
    mb.moba_check(ws)


# --- sharded forward (ranks emulated one after another: no collective) ---------------------
def _forward_keeping_idx(store):
    """A rank's forward that also keeps the GPU's selection for the oracle check."""
    def fwd(q, k, v, cu, B, topk, scale):
        out, lse, idx = mb.moba_forward(q, k, v, cu, B, topk, softmax_scale=scale,
                                        return_idx=True)
        store.append(idx)
        return out, lse
    return fwd


def test_sharded_forward_ranks_reassemble_the_forward():
    """Sequence shards: every rank's piece matches the oracle on sampled rows,
    and the pieces reassemble the unsharded forward bit for bit."""
    from block_sparse_long_11_b200 import shard
    seqlens = [4096, 12288, 3000, 9000, 650]
    w, x = synth.make_custom(seqlens, 8, 2, 128, 512, 4, seed=991, device=DEV)
    full_out, full_lse = mb.moba_forward(x["q"], x["k"], x["v"], x["cu_seqlens"], 512, 4)
    out = torch.empty_like(full_out)
    lse = torch.empty_like(full_lse)
    ranges = shard.plan_sequence_shards(seqlens, 3, 512, 4)
    for rank in range(3):
        idx = []
        t0, t1, o, l = shard.moba_forward_sharded(x["q"], x["k"], x["v"], w.seqlens, 512, 4,
                                                  rank=rank, world=3,
                                                  forward_fn=_forward_keeping_idx(idx))
        out[t0:t1] = o
        lse[t0:t1] = l
        mb.moba_check()
        torch.cuda.synchronize()
        a, b = ranges[rank]
        if t1 > t0:   # this rank's piece against the oracle, as a batch of its own
            wl = synth.Workload("rank", seqlens[a:b], 8, 2, 128, 512, 4, 0)
            xl = {"q": x["q"][t0:t1], "k": x["k"][t0:t1], "v": x["v"][t0:t1]}
            P.check_rows(xl, wl, o, l, idx[0], synth.sample_rows(wl, 384, 40 + rank))
    assert torch.equal(out, full_out) and torch.equal(lse, full_lse)


@pytest.mark.parametrize("world", [2, 4, 8])
def test_head_sharded_forward_matches_oracle_and_reassembles(world):
    """Head-group shards of one long sequence (8 query / 2 kv heads): every
    rank's heads match the oracle on sampled rows and the ranks reassemble the
    unsharded forward bit for bit."""
    from block_sparse_long_11_b200 import shard
    L, Hq, Hkv, B, topk = 20000, 8, 2, 512, 4
    w, x = synth.make_custom([L], Hq, Hkv, 128, B, topk, seed=993, device=DEV)
    full_out, full_lse = mb.moba_forward(x["q"], x["k"], x["v"], x["cu_seqlens"], B, topk)
    out = torch.empty_like(full_out)
    lse = torch.empty_like(full_lse)
    for rank in range(world):
        idx = []
        h0, h1, o, l = shard.moba_forward_head_sharded(x["q"], x["k"], x["v"], x["cu_seqlens"], B,
                                                       topk, rank=rank, world=world,
                                                       forward_fn=_forward_keeping_idx(idx))
        out[:, h0:h1] = o
        lse[:, h0:h1] = l
        mb.moba_check()
        torch.cuda.synchronize()
        _, _, g0, g1 = shard.plan_head_shards(Hq, Hkv, world)[rank]
        wl = synth.Workload("rank", [L], h1 - h0, g1 - g0, 128, B, topk, 0)
        xl = {"q": x["q"][:, h0:h1].contiguous(), "k": x["k"][:, g0:g1].contiguous(),
              "v": x["v"][:, g0:g1].contiguous()}
        P.check_rows(xl, wl, o, l, idx[0], synth.sample_rows(wl, 256, 50 + rank))
    assert torch.equal(out, full_out) and torch.equal(lse, full_lse)


# --- decode: one new token per sequence against a padded cache ---------------------------
DECODE = [
    # cache lengths (incl. the new token), max_len, Hq, Hkv, d, B, topk
    ([1, 64, 65, 700, 1500, 2048], 2048, 4, 2, 128, 64, 8),  # own block only; block end/start
    ([300, 1000, 1999], 2000, 4, 4, 64, 128, 3),              # d64
    ([5000, 4097, 3584], 6000, 8, 2, 128, 512, 4),            # GQA 4:1, B 512
    ([2560], 2560, 2, 1, 128, 64, 20),                        # top-k 20 of 40 blocks
    ([6244, 5596, 2049], 8192, 4, 2, 128, 2048, 2),           # blocks cut in 2 parts each
]


@pytest.mark.parametrize("case", DECODE, ids=[str(i) for i in range(len(DECODE))])
def test_decode_matches_prefill_row(case):
    lens, max_len, Hq, Hkv, d, B, topk = case
    x = synth.make_decode(len(lens), max_len, Hq, Hkv, d, seed=970 + len(lens), device=DEV)
    sl = torch.tensor(lens, dtype=torch.int32, device=DEV)
    kbar = mb.moba_decode_init(x["k_cache"], sl, B)
    out, lse, idx = mb.moba_decode(x["q"], x["k_cache"], x["v_cache"], sl, kbar, B, topk,
                                   return_idx=True)
    mb.moba_check()
    torch.cuda.synchronize()
    P.check_decode(x["q"], x["k_cache"], x["v_cache"], lens, out, lse, idx, B, topk)


def test_decode_steps_extend_block_means():
    """Steps across block boundaries: a block filled by a step's new token is
    averaged into the cache and scored by the next step."""
    B, topk, Hq, Hkv, d = 64, 3, 4, 2, 128
    lens = [190, 253]
    x = synth.make_decode(2, 320, Hq, Hkv, d, seed=977, device=DEV)
    sl = torch.tensor(lens, dtype=torch.int32, device=DEV)
    kbar = mb.moba_decode_init(x["k_cache"], sl, B)
    for step in range(5):   # seq 0: 191, 192 (fills block 2), 193, ...; seq 1: 254 .. 258
        lens = [L + 1 for L in lens]
        sl = torch.tensor(lens, dtype=torch.int32, device=DEV)
        q = synth.normal_bf16((2, Hq, d), 980 + step, 40, DEV)
        out, lse, idx = mb.moba_decode(q, x["k_cache"], x["v_cache"], sl, kbar, B, topk,
                                       return_idx=True)
        mb.moba_check()
        torch.cuda.synchronize()
        P.check_decode(q, x["k_cache"], x["v_cache"], lens, out, lse, idx, B, topk)
    got = kbar.cpu().numpy()
    for s, L in enumerate(lens):
        ref = R.block_means(P.bits(x["k_cache"][s, :L]), B)
        assert np.allclose(got[s, :L // B], ref, rtol=1e-6, atol=1e-7)


def test_decode_bad_seqlens():
    x = synth.make_decode(2, 256, 2, 2, 64, seed=5, device=DEV)
    sl = torch.tensor([100, 300], dtype=torch.int32, device=DEV)   # 300 > max_len
    kbar = mb.decode_kbar_cache(x["k_cache"], 64)
    ws = mb.Workspace()
    mb.moba_decode(x["q"], x["k_cache"], x["v_cache"], sl, kbar, 64, 3, workspace=ws)
    with pytest.raises(mb.MobaError) as ei:
        mb.moba_check(ws)
    assert ei.value.code == 6


# --- benchmark workloads at full size, sampled rows -----------------------------------
def _full(name, n_rows, seed):
    w = synth.WORKLOADS[name]
    x = synth.make_inputs(w, DEV)
    out, lse, idx = _run(w, x)
    rows = synth.sample_rows(w, n_rows, seed)
    return w, x, out, lse, idx, rows


def test_scaling_4x8k_h16_b512_sampled():
    w, x, out, lse, idx, rows = _full("scaling_4x8k_h16_b512", 2048, 11)
    P.check_rows(x, w, out, lse, idx, rows)


def test_needle_2x32k_h16_b512_sampled_and_recall():
    w, x, out, lse, idx, rows = _full("needle_2x32k_h16_b512", 1024, 12)
    needle_rows = []
    hit = tot = 0
    cu = w.cu_seqlens()
    g = idx.cpu().numpy()
    for nd in x["meta"]["needles"]:
        for t in nd["positions"]:
            tg = cu[nd["seq"]] + t
            hit += nd["block"] in g[tg, nd["head"]]
            tot += 1
            if len(needle_rows) < 512 and tot % 3 == 0:
                needle_rows.append((tg, nd["head"]))
    assert hit / tot >= 0.97, (hit, tot)
    P.check_rows(x, w, out, lse, idx, sorted(set(rows) | set(needle_rows)))


def test_varlen_377k_gqa32x8_b4096_sampled():
    w, x, out, lse, idx, rows = _full("varlen_377k_gqa32x8_b4096", 1024, 13)
    P.check_rows(x, w, out, lse, idx, rows)


def test_long_1m_gqa32x8_b4096_sampled():
    """4096 seeded stratified rows of the 1M-token workload."""
    w, x, out, lse, idx, rows = _full("long_1m_gqa32x8_b4096", 4096, 14)
    st = P.check_rows(x, w, out, lse, idx, rows, threads=8)
    assert st["rows"] == 4096
    assert torch.isfinite(lse).all()


def test_long_10m_gqa8x2_b4096_sampled():
    """4096 seeded stratified rows of the 10M-token workload."""
    w, x, out, lse, idx, rows = _full("long_10m_gqa8x2_b4096", 4096, 15)
    st = P.check_rows(x, w, out, lse, idx, rows, threads=8)
    assert st["rows"] == 4096
    assert torch.isfinite(lse).all()


# --- failure path: a bounded wait that runs out ------------------------------------------
def test_attention_wait_runs_out_then_workspace_runs_clean():
    """In the library's wait test mode the attention kernel's Q-gather warps
    publish no work, so the other roles' first waits (before any copy or
    tensor-core instruction) run out: moba_check must report MOBA_ERR_TIMEOUT.
    The same workspace then runs a normal forward that matches the oracle."""
    w, x = synth.make_custom([1500, 700], 4, 2, 128, 128, 4, seed=777, device=DEV)
    ws = mb.Workspace()
    L = mb.lib()
    L.moba_debug_attention_wait_test(1)
    try:
        mb.moba_forward(x["q"], x["k"], x["v"], x["cu_seqlens"], w.block_size, w.topk,
                        workspace=ws)
        with pytest.raises(mb.MobaError) as ei:
            mb.moba_check(ws)
        assert ei.value.code == 5   # MOBA_ERR_TIMEOUT
    finally:
        L.moba_debug_attention_wait_test(0)
    out, lse, idx = mb.moba_forward(x["q"], x["k"], x["v"], x["cu_seqlens"], w.block_size, w.topk,
                                    workspace=ws, return_idx=True)
    mb.moba_check(ws)
    torch.cuda.synchronize()
    P.check_rows(x, w, out, lse, idx, P.all_rows(w))
