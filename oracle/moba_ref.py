"""CPU oracle for the MoBA causal prefill forward.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module.  The
product path (the C-ABI library and its Python binding) never calls it and
has no CPU fallback.

It is a plain, slow, fp64 restatement of what the method computes, written
from these pages (cited by title and section):

  [W] the MoBA write-up "同一天，DeepSeek和月之暗面發表了關于改進注意力機制的論文"
      (senqingzn.com): sections "MoBA：將 MoE 原理應用于注意力機制" (block
      partition, parameter-free top-k gate, the five implementation steps),
      "大語言模型評估" (block 4096, top-k 12, 95.31% sparsity, 62.5% on RULER).
  [S] the summary page of arXiv 2502.13189 "MoBA: Mixture of Block Attention
      for Long-Context LLMs" (aipaper.jasonlin.tech): "Key contributions"
      (seamless full <-> sparse switch), section list ("2.1 Preliminaries:
      Standard Attention in Transformer").
  [E] the explainer "月球計畫 AI 研究介紹混合區塊注意力 (MoBA)：一種將混合專家
      (MoE) 原則應用於注意力機制的新 AI 方法" (taiwanai.tw), section
      "技術細節與優勢": the gate compares the query with an aggregated
      representation of each block's keys, keeps the best-scoring blocks, always
      includes the query's own block and enforces the causal mask.

Readings taken where the pages are silent (each listed in the design notes):
  (i)   the aggregate is the arithmetic mean of the block's keys;
  (ii)  the score is the unscaled dot product q . Kbar (a positive scale does
        not change a top-k);
  (iii) the own block counts inside k: k - 1 past blocks plus the own block;
  (iv)  equal scores break toward the lower block index;
  (v)   with grouped heads each query head routes on its own, against the mean
        keys of its KV head (h // (Hq / Hkv));
  (vi)  softmax scale 1/sqrt(d) unless given;  (vii) lse is the natural log of
        the sum of exp(scaled logits);
  (viii) blocks restart at each sequence start; a short last block is only ever
        some query's own block, so only full blocks get a mean and a score;
  (ix)  selected indices are reported ascending, padded with -1.

Parity status: every function here is pinned by tests that do not re-type its
formulas (brute-force loops, library special cases, closed forms and the
pages' printed sparsities; for the backward, central finite differences of
the forward, fp64 autograd of causal attention, and the identities
sum_u dv_u = sum dout, sum_u dk_u = 0); see the oracle test modules.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

TIE_REL = 1e-4


# --------------------------------------------------------------------------
# value conversion
# --------------------------------------------------------------------------
def as_f64(x) -> np.ndarray:
    """Exact fp64 view of an array of bf16 values.

    ``uint16`` arrays are read as bf16 bit patterns (bf16 is the top half of an
    fp32); float32/float64 arrays must already hold bf16-representable values.
    """
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


# --------------------------------------------------------------------------
# [E] 技術細節與優勢 / [W] MoBA section: block partition and aggregate keys
# --------------------------------------------------------------------------
def n_blocks(L: int, B: int) -> int:
    """Blocks covering a sequence of L tokens (the last one may be short)."""
    return (L + B - 1) // B


def block_means(k_seq, B: int) -> np.ndarray:
    """Mean key of every FULL block of one sequence.

    k_seq: [L, Hkv, d] (bf16 values as uint16 bits or floats).
    Returns Kbar [floor(L/B), Hkv, d] in fp64.  Reading (i): the "aggregated
    representation" of a block's keys is their arithmetic mean.
    """
    L = k_seq.shape[0]
    nfull = L // B
    out = np.empty((nfull,) + tuple(k_seq.shape[1:]), dtype=np.float64)
    for i in range(nfull):
        out[i] = as_f64(k_seq[i * B:(i + 1) * B]).mean(axis=0)
    return out


# --------------------------------------------------------------------------
# [W] parameter-free top-k gate; [E] own block always in, no future blocks
# --------------------------------------------------------------------------
def gate_scores(q_row, kbar_g: np.ndarray, j: int) -> np.ndarray:
    """Affinity of one query with each past block i < j: q . Kbar_i.

    Computed in fp64 and rounded to fp32 ("fp32 gate scores").  Blocks i >= j
    are never scored: the own block j is forced and later blocks are in the
    future (causal block mask).
    """
    q = as_f64(q_row)
    s = kbar_g[:j] @ q
    return s.astype(np.float32)


def select_blocks(scores: np.ndarray, j: int, topk: int):
    """Selected blocks of a query in block j, and whether the cut is a near-tie.

    The own block j is always selected and counted inside topk (reading iii);
    the other topk-1 are the best past scores, ties to the lower index
    (reading iv).  With j + 1 <= topk every block 0..j is selected.
    Returns (ascending list of block indices, tie flag).  The tie flag is set
    when the last kept and the first dropped past score differ by less than
    1e-4 of the larger magnitude: there several selections are correct.
    """
    if j + 1 <= topk:
        return list(range(j + 1)), False
    order = sorted(range(j), key=lambda i: (-float(scores[i]), i))
    kept = order[:topk - 1]
    a = float(scores[order[topk - 2]]) if topk >= 2 else None
    b = float(scores[order[topk - 1]]) if topk - 1 < j else None
    tie = False
    if a is not None and b is not None:
        tie = abs(a - b) < TIE_REL * max(abs(a), abs(b))
    return sorted(kept + [j]), tie


def moba_mask_row(sel: Sequence[int], t: int, L: int, B: int, keys=None) -> np.ndarray:
    """Explicit boolean key mask of the query at in-sequence position t.

    Key u (in-sequence) is attended iff its block u // B is selected and u <= t
    (token-level causal mask, which only bites inside the own block).  The mask
    is evaluated over every key 0..L-1, or only over the given key indices
    (``keys``): the predicate is the same, the caller just skips keys it knows
    to be outside every selected block.
    """
    u = np.arange(L) if keys is None else np.asarray(keys, dtype=np.int64)
    in_sel = np.isin(u // B, np.asarray(list(sel), dtype=np.int64))
    return in_sel & (u <= t)


def selected_block_keys(sel: Sequence[int], L: int, B: int) -> np.ndarray:
    """Ascending indices of every key inside the selected blocks (clipped to
    the sequence end): the only keys a row's mask can let through."""
    parts = [np.arange(i * B, min((i + 1) * B, L)) for i in sorted(set(int(i) for i in sel))]
    return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)


# --------------------------------------------------------------------------
# [S] 2.1 standard attention, restricted to the mask; [W] step 5 (online
# softmax merge) is written out separately in lse_merge.
# --------------------------------------------------------------------------
def attend_row(q_row, k_g, v_g, mask: np.ndarray, scale: float):
    """softmax(scale * q k^T | mask) v and its log-sum-exp, in fp64.

    k_g, v_g: [L, d] keys and values of the query's KV head.  Masked keys have
    weight exactly 0, so only the mask's keys enter the sums.
    Returns (o [d], lse) with lse = ln sum_u exp(scale * q . k_u).
    """
    keys = np.flatnonzero(mask)
    q = as_f64(q_row)
    kk = as_f64(k_g[keys])
    vv = as_f64(v_g[keys])
    logits = scale * (kk @ q)
    m = logits.max()
    p = np.exp(logits - m)
    z = p.sum()
    return (p @ vv) / z, m + math.log(z)


def lse_merge(parts):
    """Merge partial attention results over disjoint key sets.

    parts: iterable of (o_i, lse_i), each o_i normalised over its own keys.
    Returns (o, lse) equal to attention over the union of the key sets:
    m = max lse_i, w_i = exp(lse_i - m), o = sum w_i o_i / sum w_i,
    lse = m + ln sum w_i  ([W] step 5: merge by online softmax).
    """
    parts = list(parts)
    m = max(p[1] for p in parts)
    w = np.array([math.exp(p[1] - m) for p in parts])
    o = sum(wi * np.asarray(p[0], dtype=np.float64) for wi, p in zip(w, parts)) / w.sum()
    return o, m + math.log(w.sum())


# --------------------------------------------------------------------------
# whole forward
# --------------------------------------------------------------------------
def _default_scale(d: int, scale: Optional[float]) -> float:
    return 1.0 / math.sqrt(d) if (scale is None or scale <= 0) else float(scale)


def forward_rows(q_rows, t_local, heads, k_seq, v_seq, n_heads: int, n_kv_heads: int,
                 B: int, topk: int, scale: Optional[float] = None, kbar=None,
                 sel_override=None):
    """Oracle forward for chosen (position, head) rows of ONE sequence.

    q_rows: [R, d] query vectors; t_local: [R] in-sequence positions;
    heads: [R] query heads; k_seq, v_seq: [L, Hkv, d] of that sequence.
    kbar: optional precomputed block_means(k_seq, B).
    sel_override: optional list of R selections (e.g. the GPU's), used in
    place of the gate to judge attention at near-ties.
    Returns dict(out [R, d], lse [R], sel [list], tie [R] bool).
    """
    L, _, d = k_seq.shape
    G = n_heads // n_kv_heads
    scale = _default_scale(d, scale)
    if kbar is None:
        kbar = block_means(k_seq, B)
    R = len(t_local)
    out = np.zeros((R, d))
    lse = np.zeros(R)
    sels, ties = [], np.zeros(R, dtype=bool)
    for r in range(R):
        t, h = int(t_local[r]), int(heads[r])
        g = h // G
        j = t // B
        if sel_override is not None:
            sel, tie = list(sel_override[r]), False
        else:
            sc = gate_scores(q_rows[r], kbar[:, g, :], j)
            sel, tie = select_blocks(sc, j, topk)
        # the mask is evaluated over the selected blocks' keys only (every
        # other key is outside the mask), so long sequences cost O(k B) per row
        cand = selected_block_keys(sel, L, B)
        mask = moba_mask_row(sel, t, L, B, keys=cand)
        o, l = attend_row(q_rows[r], k_seq[cand, g, :], v_seq[cand, g, :], mask, scale)
        out[r], lse[r] = o, l
        sels.append(sel)
        ties[r] = tie
    return {"out": out, "lse": lse, "sel": sels, "tie": ties}


def forward(q, k, v, cu_seqlens, n_heads: int, n_kv_heads: int, B: int, topk: int,
            scale: Optional[float] = None):
    """Oracle forward for every row of a packed varlen batch (small inputs).

    q: [T, Hq, d], k, v: [T, Hkv, d], cu_seqlens: [n_seqs + 1].
    Returns dict(out [T, Hq, d], lse [T, Hq], idx [T, Hq, topk] int32 ascending
    with -1 padding, tie [T, Hq] bool).
    """
    q = np.asarray(q)
    cu = [int(c) for c in np.asarray(cu_seqlens)]
    T, Hq, d = q.shape
    out = np.zeros((T, Hq, d))
    lse = np.zeros((T, Hq))
    idx = np.full((T, Hq, topk), -1, dtype=np.int32)
    tie = np.zeros((T, Hq), dtype=bool)
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        if b <= a:
            continue
        ks, vs = k[a:b], v[a:b]
        kbar = block_means(ks, B)
        L = b - a
        tl = np.repeat(np.arange(L), Hq)
        hh = np.tile(np.arange(Hq), L)
        res = forward_rows(q[a:b].reshape(L * Hq, d), tl, hh, ks, vs, n_heads, n_kv_heads,
                           B, topk, scale, kbar=kbar)
        out[a:b] = res["out"].reshape(L, Hq, d)
        lse[a:b] = res["lse"].reshape(L, Hq)
        tie[a:b] = res["tie"].reshape(L, Hq)
        for r, sel in enumerate(res["sel"]):
            idx[a + r // Hq, r % Hq, :len(sel)] = sel
    return {"out": out, "lse": lse, "idx": idx, "tie": tie}


# --------------------------------------------------------------------------
# Backward of the forward above with the selection held fixed ([W] opening
# list: "trainable block-sparse attention" -- the blocks are chosen by the
# top-k, which passes no gradient; the attention over the chosen keys is
# ordinary softmax attention, so its derivative is that of attend_row).
# --------------------------------------------------------------------------
def attend_row_grad(q_row, k_g, v_g, mask: np.ndarray, scale: float, dout_row):
    """Derivative of attend_row's output o (for an upstream gradient dout) with
    respect to q, the masked-in keys and their values, in fp64.

    With p = softmax(scale * q k^T) over the masked keys and o = p v:
      dv_u = p_u dout,  dp_u = dout . v_u,  D = dout . o,
      ds_u = p_u (dp_u - D),  dq = scale sum_u ds_u k_u,  dk_u = scale ds_u q.
    Returns (dq [d], keys [n], dk [n, d], dv [n, d]).
    """
    keys = np.flatnonzero(mask)
    q = as_f64(q_row)
    kk = as_f64(k_g[keys])
    vv = as_f64(v_g[keys])
    g = np.asarray(dout_row, dtype=np.float64)
    logits = scale * (kk @ q)
    p = np.exp(logits - logits.max())
    p /= p.sum()
    o = p @ vv
    dv = np.outer(p, g)
    dp = vv @ g
    ds = p * (dp - g @ o)
    dq = scale * (ds @ kk)
    dk = scale * np.outer(ds, q)
    return dq, keys, dk, dv


def backward(q, k, v, cu_seqlens, dout, n_heads: int, n_kv_heads: int, B: int, topk: int,
             scale: Optional[float] = None, idx=None):
    """Gradients (dq, dk, dv) of sum(dout * out) for a packed varlen batch.

    The selection is the oracle gate's unless idx [T, Hq, topk] (ascending,
    -1 padded, e.g. a forward's own selection) is given.  Each kv head's dk,
    dv sum the contributions of every query head of its group.  fp64.
    """
    q = np.asarray(q)
    cu = [int(c) for c in np.asarray(cu_seqlens)]
    T, Hq, d = q.shape
    Hkv = n_kv_heads
    G = n_heads // n_kv_heads
    sc = _default_scale(d, scale)
    dq = np.zeros((T, Hq, d))
    dk = np.zeros((T, Hkv, d))
    dv = np.zeros((T, Hkv, d))
    dout = np.asarray(dout, dtype=np.float64)
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        if b <= a:
            continue
        ks, vs = k[a:b], v[a:b]
        kbar = block_means(ks, B)
        L = b - a
        for t in range(L):
            j = t // B
            for h in range(Hq):
                g = h // G
                if idx is not None:
                    sel = [int(x) for x in np.asarray(idx)[a + t, h] if x >= 0]
                else:
                    sel, _ = select_blocks(gate_scores(q[a + t, h], kbar[:, g, :], j), j, topk)
                mask = moba_mask_row(sel, t, L, B)
                gq, keys, gk, gv = attend_row_grad(q[a + t, h], ks[:, g, :], vs[:, g, :], mask,
                                                   sc, dout[a + t, h])
                dq[a + t, h] = gq
                dk[a + keys, g] += gk
                dv[a + keys, g] += gv
    return {"dq": dq, "dk": dk, "dv": dv}


def attend_row_grad_saved(q_row, k_g, v_g, mask, scale: float, dout_row, lse_row, out_row):
    """attend_row_grad from the forward's saved statistics, as a backward pass
    receives them: p_u = exp(scale * q . k_u - lse) and D = dout . out, with
    lse and out the forward's (here: given values, e.g. rounded to the
    precision the forward stores them in).  With the exact lse and out this is
    the same derivative.  Also returns, for error budgets, the sums of the
    absolute values of the terms of each result:
      |dq| <= scale sum_u |ds_u| |k_u|,  |dk_u| <= scale |ds_u| |q|,
      |dv_u| <= p_u |dout|.
    Returns (dq, keys, dk, dv, dq_abs, dk_abs, dv_abs)."""
    keys = np.flatnonzero(mask)
    q = as_f64(q_row)
    kk = as_f64(k_g[keys])
    vv = as_f64(v_g[keys])
    g = np.asarray(dout_row, dtype=np.float64)
    p = np.exp(scale * (kk @ q) - float(lse_row))
    dp = vv @ g
    D = float(g @ np.asarray(out_row, dtype=np.float64))
    ds = p * (dp - D)
    dq = scale * (ds @ kk)
    dk = scale * np.outer(ds, q)
    dv = np.outer(p, g)
    dq_abs = scale * (np.abs(ds) @ np.abs(kk))
    dk_abs = scale * np.outer(np.abs(ds), np.abs(q))
    dv_abs = np.outer(p, np.abs(g))
    return dq, keys, dk, dv, dq_abs, dk_abs, dv_abs


def backward_saved(q, k, v, cu_seqlens, dout, out, lse, idx, n_heads: int, n_kv_heads: int,
                   B: int, topk: int, scale: Optional[float] = None):
    """backward() with the forward's saved out [T, Hq, d] and lse [T, Hq] given
    (attend_row_grad_saved) and the selection idx.  Returns dq, dk, dv and the
    matching absolute-term sums dq_abs, dk_abs, dv_abs (fp64)."""
    q = np.asarray(q)
    cu = [int(c) for c in np.asarray(cu_seqlens)]
    T, Hq, d = q.shape
    Hkv = n_kv_heads
    G = n_heads // n_kv_heads
    sc = _default_scale(d, scale)
    res = {n: np.zeros((T, Hq if n.startswith("dq") else Hkv, d))
           for n in ("dq", "dk", "dv", "dq_abs", "dk_abs", "dv_abs")}
    dout = np.asarray(dout, dtype=np.float64)
    out = np.asarray(out, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    idx = np.asarray(idx)
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        if b <= a:
            continue
        ks, vs = k[a:b], v[a:b]
        L = b - a
        for t in range(L):
            for h in range(Hq):
                g = h // G
                sel = [int(x) for x in idx[a + t, h] if x >= 0]
                cand = selected_block_keys(sel, L, B)
                mask = moba_mask_row(sel, t, L, B, keys=cand)
                gq, kidx, gk, gv, aq, ak, av = attend_row_grad_saved(
                    q[a + t, h], ks[cand, g, :], vs[cand, g, :], mask, sc, dout[a + t, h],
                    lse[a + t, h], out[a + t, h])
                keys = cand[kidx]
                res["dq"][a + t, h] = gq
                res["dq_abs"][a + t, h] = aq
                res["dk"][a + keys, g] += gk
                res["dv"][a + keys, g] += gv
                res["dk_abs"][a + keys, g] += ak
                res["dv_abs"][a + keys, g] += av
    return res


def backward_saved_sample(q, k, v, cu_seqlens, dout, out, lse, idx, n_heads: int,
                          n_kv_heads: int, B: int, topk: int, rows=(), keys=(),
                          scale: Optional[float] = None):
    """backward_saved at a sample, for inputs too large to differentiate whole:
    dq and dq_abs of the query rows ``rows`` [(token, head)], and dk, dv,
    dk_abs, dv_abs of the keys ``keys`` [(token, kv head)].  Each comes from
    its own definition.  A row's dq is attend_row_grad_saved over the keys it
    attends.  A key's dk, dv sum, over every row that attends the key -- rows
    (t, h) of the key's sequence with h in the kv head's group, the key's
    block among the row's selected blocks and t at or after the key (the
    causal mask inside the own block; a past block lies wholly before t) --
    that row's terms for the key, as attend_row_grad_saved forms them:
      p = exp(scale q.k - lse), ds = p (dout . v - D), D = dout . out,
      dk += scale ds q, dv += p dout   (abs sums: scale |ds| |q|, p |dout|).
    Arrays may be bf16 bit patterns (uint16); only the rows read are
    converted.  Returns a dict of fp64 arrays, one row per sample entry."""
    cu = [int(c) for c in np.asarray(cu_seqlens)]
    Hq, Hkv = n_heads, n_kv_heads
    G = Hq // Hkv
    d = np.asarray(q[0, 0]).shape[-1]
    sc = _default_scale(d, scale)
    idx = np.asarray(idx)
    lse = np.asarray(lse, dtype=np.float64)

    def seq_of(t):
        s = int(np.searchsorted(cu, t, side="right")) - 1
        return s, cu[s], cu[s + 1] - cu[s]

    res = {"dq": np.zeros((len(rows), d)), "dq_abs": np.zeros((len(rows), d))}
    for i, (t, h) in enumerate(rows):
        _, a, L = seq_of(t)
        g = h // G
        sel = [int(x) for x in idx[t, h] if x >= 0]
        cand = selected_block_keys(sel, L, B)
        mask = moba_mask_row(sel, t - a, L, B, keys=cand)
        gq, _, _, _, aq, _, _ = attend_row_grad_saved(
            q[t, h], k[a + cand, g, :], v[a + cand, g, :], mask, sc,
            as_f64(dout[t, h]), lse[t, h], as_f64(out[t, h]))
        res["dq"][i], res["dq_abs"][i] = gq, aq
    for n in ("dk", "dv", "dk_abs", "dv_abs"):
        res[n] = np.zeros((len(keys), d))
    for i, (u, g) in enumerate(keys):
        _, a, L = seq_of(u)
        jb = (u - a) // B
        kv = as_f64(k[u, g])
        vv = as_f64(v[u, g])
        for h in range(g * G, (g + 1) * G):
            # rows at or after the key whose selection holds the key's block
            ts = u + np.flatnonzero((idx[u:a + L, h] == jb).any(axis=1))
            if ts.size == 0:
                continue
            qr = as_f64(q[ts, h])
            gr = as_f64(dout[ts, h])
            D = np.sum(gr * as_f64(out[ts, h]), axis=1)
            p = np.exp(sc * (qr @ kv) - lse[ts, h])
            ds = p * (gr @ vv - D)
            res["dk"][i] += sc * (ds @ qr)
            res["dv"][i] += p @ gr
            res["dk_abs"][i] += sc * (np.abs(ds) @ np.abs(qr))
            res["dv_abs"][i] += p @ np.abs(gr)
    return res


# --------------------------------------------------------------------------
# closed forms the pages fix
# --------------------------------------------------------------------------
def attended_keys(t: int, B: int, topk: int) -> int:
    """Keys attended by the query at in-sequence position t.

    Its own block contributes t - jB + 1 keys (causal), and min(topk-1, j)
    past blocks contribute B keys each (every past block is full).
    """
    j = t // B
    return (t - j * B + 1) + min(topk - 1, j) * B


def sparsity_last_query(L: int, B: int, topk: int) -> float:
    """Fraction of a length-L context that the last query does NOT attend.

    For block-aligned L this is 1 - topk*B/L, the figure the pages quote
    (95.31% at block 4096, top-k 12, 1M tokens; 62.5% at 128K).
    """
    return 1.0 - attended_keys(L - 1, B, topk) / L


def causal_avg_sparsity(L: int, B: int, topk: int) -> float:
    """1 - (attended key pairs) / (causal key pairs) over a length-L sequence."""
    att = 0
    for t in range(L):
        att += attended_keys(t, B, topk)
    return 1.0 - att / (L * (L + 1) / 2)


def total_flops(seqlens, n_heads: int, head_dim: int, B: int, topk: int) -> int:
    """Algorithmic flops 4 * d * sum over (t, h) of attended keys (QK^T and PV)."""
    total = 0
    for L in seqlens:
        L = int(L)
        nb = (L + B - 1) // B
        keys = 0
        for j in range(nb):
            lo, hi = j * B, min(L, (j + 1) * B)
            n = hi - lo
            # own block: sum_{u=1..n} u ; past blocks: n * min(topk-1, j) * B
            keys += n * (n + 1) // 2 + n * min(topk - 1, j) * B
        total += 4 * head_dim * keys * n_heads
    return total


# --------------------------------------------------------------------------
# brute force (tiny inputs only): loops, no vector library calls
# --------------------------------------------------------------------------
def brute_force(q, k, v, cu_seqlens, n_heads: int, n_kv_heads: int, B: int, topk: int,
                scale: Optional[float] = None):
    """Loop-only restatement of the whole forward for tiny inputs.

    Independent of the vectorised path above: means are summed key by key,
    the top-k is taken by repeated arg-max, the mask is an if-chain per key,
    and the softmax uses two explicit passes.  Returns (out, lse, idx) as lists.
    """
    qf = as_f64(q)
    kf = as_f64(k)
    vf = as_f64(v)
    T, Hq, d = qf.shape
    G = n_heads // n_kv_heads
    sc = 1.0 / math.sqrt(d) if (scale is None or scale <= 0) else float(scale)
    cu = [int(c) for c in np.asarray(cu_seqlens)]
    out = [[[0.0] * d for _ in range(Hq)] for _ in range(T)]
    lse = [[0.0] * Hq for _ in range(T)]
    idx = [[[-1] * topk for _ in range(Hq)] for _ in range(T)]
    for s in range(len(cu) - 1):
        a, L = cu[s], cu[s + 1] - cu[s]
        for h in range(Hq):
            g = h // G
            nfull = L // B
            means = []
            for i in range(nfull):
                m = [0.0] * d
                for u in range(i * B, (i + 1) * B):
                    for c in range(d):
                        m[c] += kf[a + u, g, c]
                means.append([x / B for x in m])
            for t in range(L):
                j = t // B
                scores = {}
                for i in range(j):
                    acc = 0.0
                    for c in range(d):
                        acc += qf[a + t, h, c] * means[i][c]
                    scores[i] = float(np.float32(acc))
                chosen = [j]
                left = dict(scores)
                while len(chosen) < topk and left:
                    best = None
                    for i in sorted(left):
                        if best is None or left[i] > left[best]:
                            best = i
                    chosen.append(best)
                    del left[best]
                chosen.sort()
                for p, i in enumerate(chosen):
                    idx[a + t][h][p] = i
                keys = []
                for u in range(L):
                    ok = False
                    for i in chosen:
                        if i * B <= u < (i + 1) * B:
                            ok = True
                    if u > t:
                        ok = False
                    if ok:
                        keys.append(u)
                logits = []
                for u in keys:
                    acc = 0.0
                    for c in range(d):
                        acc += qf[a + t, h, c] * kf[a + u, g, c]
                    logits.append(sc * acc)
                mx = max(logits)
                den = 0.0
                for x in logits:
                    den += math.exp(x - mx)
                o = [0.0] * d
                for x, u in zip(logits, keys):
                    w = math.exp(x - mx) / den
                    for c in range(d):
                        o[c] += w * vf[a + u, g, c]
                out[a + t][h] = o
                lse[a + t][h] = mx + math.log(den)
    return out, lse, idx
