"""Helpers of the GPU parity tests: compare the CUDA path with the CPU oracle.

Expected values come only from ``oracle.moba_ref`` on the same bf16 bits the
GPU saw.  Tolerances (bf16 inputs, fp32 accumulation):
  * block selections bit-exact, except rows whose oracle cut is a near-tie
    (last kept and first dropped past score within 1e-4 relative); there the
    GPU's selection must still be one of the correct ones: every past block it
    keeps scores at least the oracle's cut score minus the band, every past
    block it drops scores at most the cut plus the band;
  * outputs against the oracle run on the GPU's own selection:
    max |diff| <= 1e-2 and mean |diff| <= 1e-3;
  * lse max |diff| <= 1e-3.
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

from oracle import moba_ref as R

OUT_MAX_ABS = 1e-2
OUT_MEAN_ABS = 1e-3
LSE_MAX_ABS = 1e-3


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host)."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def valid_selection(scores, j: int, topk: int, gs) -> bool:
    """Is the ascending selection gs a correct selection for a row in block j
    whose oracle (fp32) past scores are ``scores``?

    It must hold the own block j and min(topk - 1, j) distinct past blocks.
    With c = the (topk-1)-th largest past score and the next one c', and the
    band delta = 1e-4 * max(|c|, |c'|) (the oracle's near-tie width), every
    kept past block must score >= c - delta and every dropped one <= c +
    delta: a selection that swaps blocks inside the band is correct, one that
    keeps a clearly worse block or drops a clearly better one is not.
    """
    gs = list(gs)
    if j not in gs or len(set(gs)) != len(gs) or any(not (0 <= v <= j) for v in gs):
        return False
    past = [v for v in gs if v != j]
    if len(past) != min(topk - 1, j):
        return False
    if topk - 1 >= j:
        return True
    srt = np.sort(np.asarray(scores[:j], dtype=np.float64))[::-1]
    c = float(srt[topk - 2]) if topk >= 2 else float("inf")
    c_next = float(srt[topk - 1])
    if topk < 2:
        return True
    band = R.TIE_REL * max(abs(c), abs(c_next))
    keep = set(past)
    for i in range(j):
        s_i = float(scores[i])
        if i in keep and s_i < c - band:
            return False
        if i not in keep and s_i > c + band:
            return False
    return True


def _oracle_rows(q_rows, t_loc, hh, ks, vs, Hq, Hkv, B, topk, scale, kbar, sel, threads):
    """forward_rows over row batches in a thread pool (NumPy releases the GIL in
    the gathers, exps and matmuls that dominate long rows)."""
    n = len(t_loc)
    if threads <= 1 or n < 64:
        return R.forward_rows(q_rows, t_loc, hh, ks, vs, Hq, Hkv, B, topk, scale=scale, kbar=kbar,
                              sel_override=sel)
    step = -(-n // (4 * threads))
    parts = [(a, min(n, a + step)) for a in range(0, n, step)]
    with ThreadPoolExecutor(threads) as ex:
        res = list(ex.map(lambda ab: R.forward_rows(
            q_rows[ab[0]:ab[1]], t_loc[ab[0]:ab[1]], hh[ab[0]:ab[1]], ks, vs, Hq, Hkv, B, topk,
            scale=scale, kbar=kbar, sel_override=sel[ab[0]:ab[1]]), parts))
    return {"out": np.concatenate([r["out"] for r in res]),
            "lse": np.concatenate([r["lse"] for r in res])}


def check_rows(x, w, out, lse, idx, rows, kbar_cache=None, out_rtol=0.0, scale=None, threads=1):
    """Compare GPU results with the oracle on the given (t_global, h) rows.

    x: inputs dict (q, k, v on the GPU), w: the Workload, out/lse/idx: GPU
    results.  Returns a dict of statistics; raises AssertionError on failure.
    """
    cu = w.cu_seqlens()
    B, topk, Hq, Hkv = w.block_size, w.topk, w.n_heads, w.n_kv_heads
    G = Hq // Hkv
    rows = sorted(rows)
    t_idx = torch.tensor([r[0] for r in rows], dtype=torch.long, device=x["q"].device)
    h_idx = torch.tensor([r[1] for r in rows], dtype=torch.long, device=x["q"].device)
    q_rows = bits(x["q"][t_idx, h_idx])
    g_out = out[t_idx, h_idx].float().cpu().numpy()
    g_lse = lse[t_idx, h_idx].cpu().numpy().astype(np.float64)
    g_idx = idx[t_idx, h_idx].cpu().numpy()
    stats = {"rows": len(rows), "ties": 0, "sel_mismatch": 0, "max_abs": 0.0, "sum_abs": 0.0,
             "n": 0, "lse_max_abs": 0.0}
    seq_of = np.searchsorted(np.asarray(cu), [r[0] for r in rows], side="right") - 1
    for s in sorted(set(seq_of.tolist())):
        sel_rows = [i for i in range(len(rows)) if seq_of[i] == s]
        a, b = cu[s], cu[s + 1]
        ks = bits(x["k"][a:b])
        vs = bits(x["v"][a:b])
        kbar = kbar_cache.get(s) if kbar_cache is not None else None
        if kbar is None:
            kbar = R.block_means(ks, B)
            if kbar_cache is not None:
                kbar_cache[s] = kbar
        t_loc = [rows[i][0] - a for i in sel_rows]
        hh = [rows[i][1] for i in sel_rows]
        gpu_sel = []
        for n, i in enumerate(sel_rows):
            t, h = t_loc[n], hh[n]
            j = t // B
            sc = R.gate_scores(q_rows[i], kbar[:, h // G, :], j)
            ref_sel, tie = R.select_blocks(sc, j, topk)
            gs = [int(v) for v in g_idx[i] if v >= 0]
            assert all(int(v) == -1 for v in g_idx[i][len(gs):]), (rows[i], g_idx[i])
            assert gs == sorted(gs), (rows[i], gs)
            if tie:
                stats["ties"] += 1
                if gs != ref_sel:
                    stats["ties_swapped"] = stats.get("ties_swapped", 0) + 1
                # a near-tie may swap the cut, but only inside the band
                assert valid_selection(sc, j, topk, gs), (rows[i], gs, ref_sel)
            elif gs != ref_sel:
                stats["sel_mismatch"] += 1
            gpu_sel.append(gs)
        res = _oracle_rows(q_rows[sel_rows], t_loc, hh, ks, vs, Hq, Hkv, B, topk, scale, kbar,
                           gpu_sel, threads)
        d = np.abs(res["out"] - g_out[sel_rows])
        if out_rtol > 0:   # error budget that grows with |o| (see the caller)
            d = np.maximum(d - out_rtol * np.abs(res["out"]), 0.0)
        stats["max_abs"] = max(stats["max_abs"], float(d.max()))
        stats["sum_abs"] += float(d.sum())
        stats["n"] += d.size
        stats["lse_max_abs"] = max(stats["lse_max_abs"],
                                   float(np.abs(res["lse"] - g_lse[sel_rows]).max()))
    stats["mean_abs"] = stats["sum_abs"] / max(1, stats["n"])
    assert stats["sel_mismatch"] == 0, stats
    assert stats["max_abs"] <= OUT_MAX_ABS, stats
    assert stats["mean_abs"] <= OUT_MEAN_ABS, stats
    assert stats["lse_max_abs"] <= LSE_MAX_ABS, stats
    return stats


def all_rows(w):
    return [(t, h) for t in range(w.total_tokens) for h in range(w.n_heads)]


def check_full_rows(x, w, out, lse, rows, scale=None):
    """Dense causal attention (moba_forward_full) against the oracle run with
    every block 0..j selected for each row: the mask is then u <= t exactly.
    Same tolerances as check_rows.  Returns a dict of statistics."""
    cu = w.cu_seqlens()
    Hq, Hkv = w.n_heads, w.n_kv_heads
    Bo = 64  # oracle's block partition: irrelevant once every block is selected
    rows = sorted(rows)
    t_idx = torch.tensor([r[0] for r in rows], dtype=torch.long, device=x["q"].device)
    h_idx = torch.tensor([r[1] for r in rows], dtype=torch.long, device=x["q"].device)
    q_rows = bits(x["q"][t_idx, h_idx])
    g_out = out[t_idx, h_idx].float().cpu().numpy()
    g_lse = lse[t_idx, h_idx].cpu().numpy().astype(np.float64)
    stats = {"rows": len(rows), "max_abs": 0.0, "sum_abs": 0.0, "n": 0, "lse_max_abs": 0.0}
    seq_of = np.searchsorted(np.asarray(cu), [r[0] for r in rows], side="right") - 1
    for s in sorted(set(seq_of.tolist())):
        sel_rows = [i for i in range(len(rows)) if seq_of[i] == s]
        a, b = cu[s], cu[s + 1]
        ks = bits(x["k"][a:b])
        vs = bits(x["v"][a:b])
        t_loc = [rows[i][0] - a for i in sel_rows]
        hh = [rows[i][1] for i in sel_rows]
        every = [list(range(t // Bo + 1)) for t in t_loc]
        res = R.forward_rows(q_rows[sel_rows], t_loc, hh, ks, vs, Hq, Hkv, Bo, 1, scale=scale,
                             kbar=np.zeros((0, Hkv, ks.shape[2])), sel_override=every)
        d = np.abs(res["out"] - g_out[sel_rows])
        stats["max_abs"] = max(stats["max_abs"], float(d.max()))
        stats["sum_abs"] += float(d.sum())
        stats["n"] += d.size
        stats["lse_max_abs"] = max(stats["lse_max_abs"],
                                   float(np.abs(res["lse"] - g_lse[sel_rows]).max()))
    stats["mean_abs"] = stats["sum_abs"] / max(1, stats["n"])
    assert stats["max_abs"] <= OUT_MAX_ABS, stats
    assert stats["mean_abs"] <= OUT_MEAN_ABS, stats
    assert stats["lse_max_abs"] <= LSE_MAX_ABS, stats
    return stats


def check_decode(q, kc, vc, seqlens, out, lse, idx, B, topk, scale=None):
    """Decode step against the oracle's prefill row t = L - 1 of each
    sequence's first L cached tokens.  Selections bit-exact except near-ties;
    outputs judged on the GPU's selection, with check_rows' tolerances.
    q [n, Hq, d], kc / vc [n, max_len, Hkv, d] (GPU tensors); seqlens: list."""
    n, Hq, d = q.shape
    Hkv = kc.shape[2]
    qb = bits(q)
    g_out = out.float().cpu().numpy()
    g_lse = lse.cpu().numpy().astype(np.float64)
    g_idx = idx.cpu().numpy()
    st = {"rows": 0, "ties": 0, "max_abs": 0.0, "sum_abs": 0.0, "n": 0, "lse_max_abs": 0.0}
    for s in range(n):
        L = int(seqlens[s])
        ks = bits(kc[s, :L])
        vs = bits(vc[s, :L])
        t = L - 1
        heads = list(range(Hq))
        ref = R.forward_rows(qb[s], [t] * Hq, heads, ks, vs, Hq, Hkv, B, topk, scale=scale)
        gpu_sel = []
        kbar = R.block_means(ks, B)
        for h in heads:
            gs = [int(v) for v in g_idx[s, h] if v >= 0]
            assert all(int(v) == -1 for v in g_idx[s, h][len(gs):]), (s, h, g_idx[s, h])
            assert gs == sorted(gs) and gs[-1] == t // B, (s, h, gs)
            if ref["tie"][h]:
                st["ties"] += 1
                sc = R.gate_scores(qb[s, h], kbar[:, h // (Hq // Hkv), :], t // B)
                assert valid_selection(sc, t // B, topk, gs), (s, h, gs, ref["sel"][h])
            else:
                assert gs == list(ref["sel"][h]), (s, h, gs, ref["sel"][h])
            gpu_sel.append(gs)
        res = R.forward_rows(qb[s], [t] * Hq, heads, ks, vs, Hq, Hkv, B, topk, scale=scale,
                             kbar=np.zeros((0, Hkv, d)), sel_override=gpu_sel)
        dd = np.abs(res["out"] - g_out[s])
        st["rows"] += Hq
        st["max_abs"] = max(st["max_abs"], float(dd.max()))
        st["sum_abs"] += float(dd.sum())
        st["n"] += dd.size
        st["lse_max_abs"] = max(st["lse_max_abs"], float(np.abs(res["lse"] - g_lse[s]).max()))
    st["mean_abs"] = st["sum_abs"] / max(1, st["n"])
    assert st["max_abs"] <= OUT_MAX_ABS, st
    assert st["mean_abs"] <= OUT_MEAN_ABS, st
    assert st["lse_max_abs"] <= LSE_MAX_ABS, st
    return st
