"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each test fixes the oracle to something the pages or the mathematics fix:
brute-force loops on tiny inputs, library special cases (causal SDPA for the
full <-> sparse switch and for top-k = 1), closed forms, the sparsities the
pages print (tests/golden/pages_sparsity.txt) and invariants of the gate.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import moba_ref as R
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _np(t):
    return t.float().numpy()


def _sdpa_causal(q, k, v, G):
    """torch SDPA (fp64, CPU) with a causal mask; q [L, Hq, d], k/v [L, Hkv, d]."""
    qt = torch.from_numpy(q).double().permute(1, 0, 2)
    kt = torch.from_numpy(k).double().repeat_interleave(G, dim=1).permute(1, 0, 2)
    vt = torch.from_numpy(v).double().repeat_interleave(G, dim=1).permute(1, 0, 2)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    return o.permute(1, 0, 2).numpy()


def _textbook_causal(q, k, v, G):
    """Plain causal softmax attention with a triangular mask and logsumexp."""
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    L, Hq, d = q.shape
    out = np.zeros((L, Hq, d))
    lse = np.zeros((L, Hq))
    tri = np.tril(np.ones((L, L), dtype=bool))
    for h in range(Hq):
        g = h // G
        s = (q[:, h, :] @ k[:, g, :].T) / math.sqrt(d)
        s = np.where(tri, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        z = p.sum(axis=1, keepdims=True)
        out[:, h, :] = (p / z) @ v[:, g, :]
        lse[:, h] = (m + np.log(z))[:, 0]
    return out, lse


TINY = [
    # seqlens, Hq, Hkv, d, B, topk
    ([32], 1, 1, 4, 4, 1),
    ([32], 1, 1, 4, 4, 3),
    ([29], 2, 1, 6, 4, 2),        # ragged last block, GQA
    ([40, 23], 2, 2, 8, 8, 2),    # varlen
    ([64], 4, 2, 4, 8, 4),
    ([17, 9, 33], 2, 1, 4, 4, 5),
    ([64], 1, 1, 8, 8, 8),        # topk == number of blocks
]


@pytest.mark.parametrize("case", TINY)
def test_p1_brute_force_matches_vectorised(case):
    seqlens, Hq, Hkv, d, B, topk = case
    w, x = synth.make_custom(seqlens, Hq, Hkv, d, B, topk, seed=11 + len(seqlens) * 7 + topk)
    q, k, v = _np(x["q"]), _np(x["k"]), _np(x["v"])
    cu = x["cu_seqlens"].numpy()
    ref = R.forward(q, k, v, cu, Hq, Hkv, B, topk)
    out, lse, idx = R.brute_force(q, k, v, cu, Hq, Hkv, B, topk)
    np.testing.assert_allclose(ref["out"], np.array(out), rtol=0, atol=1e-12)
    np.testing.assert_allclose(ref["lse"], np.array(lse), rtol=0, atol=1e-12)
    np.testing.assert_array_equal(ref["idx"], np.array(idx, dtype=np.int32))


@pytest.mark.parametrize("Hq,Hkv", [(1, 1), (4, 2)])
def test_p2_seamless_switch_is_full_causal(Hq, Hkv):
    """topk >= number of blocks gives exactly full causal attention."""
    L, d, B = 256, 16, 32
    w, x = synth.make_custom([L], Hq, Hkv, d, B, 8, seed=21 + Hq)
    q, k, v = _np(x["q"]), _np(x["k"]), _np(x["v"])
    ref = R.forward(q, k, v, x["cu_seqlens"].numpy(), Hq, Hkv, B, 8)
    G = Hq // Hkv
    np.testing.assert_allclose(ref["out"], _sdpa_causal(q, k, v, G), rtol=0, atol=1e-12)
    o2, l2 = _textbook_causal(q, k, v, G)
    np.testing.assert_allclose(ref["out"], o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(ref["lse"], l2, rtol=0, atol=1e-12)


def test_p2_seamless_switch_single_2k_d64():
    """The 2048-token, head-dim-64, block-256 workload at top-k 8 = full causal."""
    w = synth.WORKLOADS["single_2k_d64_b256"]
    x = synth.make_inputs(w)
    q, k, v = _np(x["q"]), _np(x["k"]), _np(x["v"])
    rows = np.arange(0, 2048, 37)
    res = R.forward_rows(q[rows].reshape(len(rows), 64), rows, np.zeros(len(rows), int),
                         k, v, 1, 1, 256, 8)
    full = _sdpa_causal(q, k, v, 1)
    np.testing.assert_allclose(res["out"], full[rows, 0, :], rtol=0, atol=1e-12)


def test_p3_topk1_is_block_diagonal_causal():
    L, Hq, Hkv, d, B = 192, 2, 1, 8, 64
    w, x = synth.make_custom([L], Hq, Hkv, d, B, 1, seed=31)
    q, k, v = _np(x["q"]), _np(x["k"]), _np(x["v"])
    ref = R.forward(q, k, v, x["cu_seqlens"].numpy(), Hq, Hkv, B, 1)
    for j in range(L // B):
        sl = slice(j * B, (j + 1) * B)
        blk = _sdpa_causal(q[sl], k[sl], v[sl], Hq // Hkv)
        np.testing.assert_allclose(ref["out"][sl], blk, rtol=0, atol=1e-12)


def test_p4_invariants():
    seqlens, Hq, Hkv, d, B, topk = [300, 129], 4, 2, 8, 32, 3
    w, x = synth.make_custom(seqlens, Hq, Hkv, d, B, topk, seed=41)
    q, k, v = _np(x["q"]), _np(x["k"]), _np(x["v"])
    cu = w.cu_seqlens()
    for s, L in enumerate(seqlens):
        a = cu[s]
        ks, vs = k[a:a + L], v[a:a + L]
        kbar = R.block_means(ks, B)
        for t in range(0, L, 7):
            j = t // B
            for h in range(Hq):
                sc = R.gate_scores(q[a + t, h], kbar[:, h // (Hq // Hkv), :], j)
                sel, _ = R.select_blocks(sc, j, topk)
                assert j in sel                                  # own block always in
                assert all(i <= j for i in sel)                  # no future block
                assert len(sel) == min(topk, j + 1)
                assert sel == sorted(sel)
                m = R.moba_mask_row(sel, t, L, B)
                assert not m[t + 1:].any()                       # no future token
                assert m[j * B:t + 1].all()                      # own block up to t
                assert int(m.sum()) == R.attended_keys(t, B, topk)


def test_p4_mask_over_selected_block_keys_equals_full_mask():
    """The row mask evaluated over the selected blocks' keys only (what the
    oracle forward does for long sequences) lets through exactly the keys of
    the mask evaluated over the whole sequence."""
    rng = np.random.default_rng(9)
    for _ in range(300):
        B = int(rng.integers(1, 9))
        L = int(rng.integers(1, 80))
        t = int(rng.integers(0, L))
        j = t // B
        nsel = int(rng.integers(1, j + 2))
        sel = sorted(set([j] + [int(i) for i in rng.integers(0, j + 1, nsel)]))
        full = R.moba_mask_row(sel, t, L, B)
        cand = R.selected_block_keys(sel, L, B)
        part = R.moba_mask_row(sel, t, L, B, keys=cand)
        assert np.array_equal(cand[part], np.flatnonzero(full))
        assert np.all(np.diff(cand) > 0)
        assert ((cand // B)[:, None] == np.array(sel)[None, :]).any(axis=1).all()


def test_p4_topk_matches_library_sort():
    """Gate selection equals a stable library sort on (score desc, index asc)."""
    rng = np.random.default_rng(5)
    for trial in range(200):
        j = int(rng.integers(0, 40))
        topk = int(rng.integers(1, 10))
        sc = rng.standard_normal(j).astype(np.float32)
        if j > 3 and trial % 3 == 0:
            sc[int(rng.integers(0, j))] = sc[int(rng.integers(0, j))]   # exact tie
        sel, _ = R.select_blocks(sc, j, topk)
        order = np.lexsort((np.arange(j), -sc.astype(np.float64)))
        want = sorted(list(order[:max(0, topk - 1)]) + [j])
        assert sel == [int(i) for i in want]


def test_p4_exact_tie_prefers_lower_index():
    kbar = np.zeros((5, 1, 2))
    kbar[1, 0] = [1.0, 0.0]
    kbar[3, 0] = [1.0, 0.0]
    sc = R.gate_scores(np.array([1.0, 0.0], dtype=np.float32), kbar[:, 0, :], 5)
    sel, tie = R.select_blocks(sc, 5, 2)
    assert sel == [1, 5] and tie


def _read_golden():
    rows = []
    with open(os.path.join(GOLDEN, "pages_sparsity.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            B, topk, L, pct, dec = line.split()
            rows.append((int(B), int(topk), int(L), float(pct), int(dec)))
    return rows


def test_p5_sparsity_matches_pages():
    rows = _read_golden()
    assert len(rows) == 3
    for B, topk, L, pct, dec in rows:
        got = 100.0 * R.sparsity_last_query(L, B, topk)
        assert round(got, dec) == pct, (B, topk, L, got, pct)


def test_p5_sparsity_from_explicit_mask():
    """The same ratio counted off the oracle's explicit mask on a scaled-down case."""
    for (B, topk, L) in [(8, 2, 64), (16, 12, 1024), (4, 3, 100)]:
        w, x = synth.make_custom([L], 1, 1, 4, B, topk, seed=51)
        q, k = _np(x["q"]), _np(x["k"])
        kbar = R.block_means(k, B)
        t = L - 1
        sc = R.gate_scores(q[t, 0], kbar[:, 0, :], t // B)
        sel, _ = R.select_blocks(sc, t // B, topk)
        m = R.moba_mask_row(sel, t, L, B)
        assert abs((1 - m.sum() / L) - R.sparsity_last_query(L, B, topk)) < 1e-15


def test_p5_flop_count_closed_form():
    """Algorithmic flops = 4 d sum_t a(t) Hq, summed by brute force."""
    for seqlens, Hq, d, B, topk in [([100, 37], 2, 8, 16, 3), ([2048], 1, 64, 256, 3)]:
        brute = 0
        for L in seqlens:
            for t in range(L):
                brute += 4 * d * R.attended_keys(t, B, topk) * Hq
        assert R.total_flops(seqlens, Hq, d, B, topk) == brute
    # full causal at topk >= nb: 4 d Hq L(L+1)/2
    assert R.total_flops([2048], 1, 64, 256, 8) == 4 * 64 * 2048 * 2049 // 2


def test_p6_needle_recall():
    """A planted needle block is routed to by the queries that carry its direction."""
    w, x = synth.make_custom([8192], 4, 4, 32, 256, 3, seed=61, kind="needle")
    q, k = _np(x["q"]), _np(x["k"])
    kbar = R.block_means(k, 256)
    hit = tot = 0
    for nd in x["meta"]["needles"]:
        h, n = nd["head"], nd["block"]
        for t in nd["positions"]:
            sc = R.gate_scores(q[t, h], kbar[:, h, :], t // 256)
            sel, _ = R.select_blocks(sc, t // 256, 3)
            hit += n in sel
            tot += 1
    assert tot > 0 and hit / tot >= 0.97, (hit, tot)


def test_p7_lse_merge_equals_one_shot():
    rng = np.random.default_rng(7)
    L, d = 200, 8
    k = rng.standard_normal((L, d))
    v = rng.standard_normal((L, d))
    q = rng.standard_normal(d)
    full = np.ones(L, dtype=bool)
    o1, l1 = R.attend_row(q, k, v, full, 0.3)
    for _ in range(5):
        lab = rng.integers(0, 6, L)
        parts = []
        for c in rng.permutation(6):
            m = lab == c
            if m.any():
                parts.append(R.attend_row(q, k, v, m, 0.3))
        o2, l2 = R.lse_merge(parts)
        np.testing.assert_allclose(o2, o1, rtol=0, atol=1e-12)
        assert abs(l2 - l1) < 1e-12
    # lse itself against the library logsumexp
    s = 0.3 * (k @ q)
    assert abs(l1 - torch.logsumexp(torch.from_numpy(s), 0).item()) < 1e-12


def test_p8_permutation_inside_past_block():
    L, d, B, topk = 256, 8, 32, 3
    w, x = synth.make_custom([L], 1, 1, d, B, topk, seed=81)
    q, k, v = _np(x["q"]), _np(x["k"]), _np(x["v"])
    t = L - 5
    base = R.forward_rows(q[[t], 0], [t], [0], k, v, 1, 1, B, topk)
    past = [i for i in base["sel"][0] if i != t // B]
    i = past[0]
    perm = np.arange(L)
    perm[i * B:(i + 1) * B] = i * B + np.random.default_rng(8).permutation(B)
    res = R.forward_rows(q[[t], 0], [t], [0], k[perm], v[perm], 1, 1, B, topk)
    assert res["sel"] == base["sel"]
    np.testing.assert_allclose(res["out"], base["out"], rtol=0, atol=1e-12)
