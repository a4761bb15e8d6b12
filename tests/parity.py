"""Helpers of the GPU parity tests: compare the CUDA path with the CPU oracle.

Expected values come only from ``oracle.moba_ref`` on the same bf16 bits the
GPU saw.  Tolerances (bf16 inputs, fp32 accumulation):
  * block selections bit-exact, except rows whose oracle cut is a near-tie
    (last kept and first dropped past score within 1e-4 relative);
  * outputs against the oracle run on the GPU's own selection:
    max |diff| <= 1e-2 and mean |diff| <= 1e-3;
  * lse max |diff| <= 1e-3.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import moba_ref as R

OUT_MAX_ABS = 1e-2
OUT_MEAN_ABS = 1e-3
LSE_MAX_ABS = 1e-3


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host)."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def check_rows(x, w, out, lse, idx, rows, kbar_cache=None, out_rtol=0.0, scale=None):
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
                # a near-tie may swap the cut; the rest must still be a valid selection
                assert j in gs and len(gs) == len(ref_sel) and all(0 <= v <= j for v in gs)
            elif gs != ref_sel:
                stats["sel_mismatch"] += 1
            gpu_sel.append(gs)
        res = R.forward_rows(q_rows[sel_rows], t_loc, hh, ks, vs, Hq, Hkv, B, topk,
                             scale=scale, kbar=kbar, sel_override=gpu_sel)
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
        for h in heads:
            gs = [int(v) for v in g_idx[s, h] if v >= 0]
            assert all(int(v) == -1 for v in g_idx[s, h][len(gs):]), (s, h, g_idx[s, h])
            assert gs == sorted(gs) and gs[-1] == t // B, (s, h, gs)
            if ref["tie"][h]:
                st["ties"] += 1
                assert len(gs) == len(ref["sel"][h])
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
