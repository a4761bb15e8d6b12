"""Pins of the oracle's backward (the gradients of sum(dout * out) with the
selection held fixed).  CPU only.  None of them restates the formulas in
attend_row_grad: central finite differences of the oracle FORWARD, fp64
autograd of torch's causal attention (the full <-> sparse switch special
case), two identities of softmax attention, and planted slips that the pins
must catch."""
import numpy as np
import pytest
import torch

from oracle import moba_ref as R


def _case(seqlens, Hq, Hkv, d, seed):
    rng = np.random.default_rng(seed)
    T = sum(seqlens)
    q = rng.standard_normal((T, Hq, d))
    k = rng.standard_normal((T, Hkv, d))
    v = rng.standard_normal((T, Hkv, d))
    dout = rng.standard_normal((T, Hq, d))
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int64)
    return q, k, v, dout, cu


def _loss(q, k, v, cu, dout, Hq, Hkv, B, topk, idx, scale=None):
    """sum(dout * out) of the oracle forward with the selection idx held fixed."""
    tot = 0.0
    for s in range(len(cu) - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        L = b - a
        tl = np.repeat(np.arange(L), Hq)
        hh = np.tile(np.arange(Hq), L)
        sel = [[int(x) for x in idx[a + t, h] if x >= 0] for t, h in zip(tl, hh)]
        res = R.forward_rows(q[a:b].reshape(L * Hq, -1), tl, hh, k[a:b], v[a:b], Hq, Hkv, B,
                             topk, scale=scale, kbar=np.zeros((0, Hkv, q.shape[2])),
                             sel_override=sel)
        tot += float((res["out"] * dout[a:b].reshape(L * Hq, -1)).sum())
    return tot


def _check_finite_differences(seqlens=(37, 20), Hq=2, Hkv=1, d=4, B=8, topk=3, seed=3,
                              n_probe=40, scale=None):
    q, k, v, dout, cu = _case(list(seqlens), Hq, Hkv, d, seed)
    idx = R.forward(q, k, v, cu, Hq, Hkv, B, topk, scale)["idx"]
    g = R.backward(q, k, v, cu, dout, Hq, Hkv, B, topk, scale, idx=idx)
    rng = np.random.default_rng(seed + 100)
    eps = 1e-5
    for name, x, gx in (("q", q, g["dq"]), ("k", k, g["dk"]), ("v", v, g["dv"])):
        for _ in range(n_probe):
            pos = tuple(int(rng.integers(0, n)) for n in x.shape)
            old = x[pos]
            x[pos] = old + eps
            lp = _loss(q, k, v, cu, dout, Hq, Hkv, B, topk, idx, scale)
            x[pos] = old - eps
            lm = _loss(q, k, v, cu, dout, Hq, Hkv, B, topk, idx, scale)
            x[pos] = old
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - gx[pos]) <= 1e-6 * (1.0 + abs(fd)), (name, pos, fd, gx[pos])


def test_backward_matches_finite_differences_gqa_varlen():
    _check_finite_differences()


def test_backward_matches_finite_differences_grouped_heads_and_scale():
    _check_finite_differences(seqlens=(45,), Hq=4, Hkv=2, d=4, B=8, topk=2, seed=4, scale=0.3)


def test_backward_full_causal_equals_torch_autograd():
    # top-k >= blocks: full causal attention, differentiated by torch in fp64
    seqlens, Hq, Hkv, d, B = [50, 31], 4, 2, 8, 8
    q, k, v, dout, cu = _case(seqlens, Hq, Hkv, d, 5)
    g = R.backward(q, k, v, cu, dout, Hq, Hkv, B, 16)
    G = Hq // Hkv
    for s in range(len(seqlens)):
        a, b = int(cu[s]), int(cu[s + 1])
        tq = torch.tensor(q[a:b]).permute(1, 0, 2).requires_grad_(True)
        tk = torch.tensor(k[a:b]).permute(1, 0, 2).requires_grad_(True)
        tv = torch.tensor(v[a:b]).permute(1, 0, 2).requires_grad_(True)
        o = torch.nn.functional.scaled_dot_product_attention(
            tq[None], tk.repeat_interleave(G, 0)[None], tv.repeat_interleave(G, 0)[None],
            is_causal=True)[0]
        (o * torch.tensor(dout[a:b]).permute(1, 0, 2)).sum().backward()
        np.testing.assert_allclose(g["dq"][a:b], tq.grad.permute(1, 0, 2).numpy(), atol=1e-10)
        np.testing.assert_allclose(g["dk"][a:b], tk.grad.permute(1, 0, 2).numpy(), atol=1e-10)
        np.testing.assert_allclose(g["dv"][a:b], tv.grad.permute(1, 0, 2).numpy(), atol=1e-10)


def _check_identities(seed=6):
    # every row's weights sum to 1 (so its dv contributions sum to dout) and
    # its ds sum to 0 (so its dk contributions sum to 0), selection or not
    seqlens, Hq, Hkv, d, B, topk = [60, 25], 4, 2, 8, 8, 3
    q, k, v, dout, cu = _case(seqlens, Hq, Hkv, d, seed)
    g = R.backward(q, k, v, cu, dout, Hq, Hkv, B, topk)
    G = Hq // Hkv
    for s in range(len(seqlens)):
        a, b = int(cu[s]), int(cu[s + 1])
        for kv in range(Hkv):
            np.testing.assert_allclose(g["dv"][a:b, kv].sum(0),
                                       dout[a:b, kv * G:(kv + 1) * G].sum((0, 1)), atol=1e-10)
            np.testing.assert_allclose(g["dk"][a:b, kv].sum(0), 0.0, atol=1e-10)


def test_backward_identities():
    _check_identities()


# --- planted slips: each must make a pin fail -------------------------------------
_ORIG = R.attend_row_grad


def _without_D(q_row, k_g, v_g, mask, scale, dout_row):
    keys = np.flatnonzero(mask)
    q, kk, vv = R.as_f64(q_row), R.as_f64(k_g[keys]), R.as_f64(v_g[keys])
    p = np.exp(scale * (kk @ q) - (scale * (kk @ q)).max())
    p /= p.sum()
    gg = np.asarray(dout_row, dtype=np.float64)
    ds = p * (vv @ gg)                       # forgot the "- dout . o" term
    return scale * (ds @ kk), keys, scale * np.outer(ds, q), np.outer(p, gg)


def _dq_unscaled(*a):
    dq, keys, dk, dv = _ORIG(*a)
    return dq / a[4], keys, dk, dv


def _dk_from_keys(q_row, k_g, v_g, mask, scale, dout_row):
    dq, keys, dk, dv = _ORIG(q_row, k_g, v_g, mask, scale, dout_row)
    ds = dk[:, 0] / (scale * R.as_f64(q_row)[0])
    return dq, keys, scale * np.outer(ds, R.as_f64(k_g[keys]).mean(0)), dv


def _dv_uniform(*a):
    dq, keys, dk, dv = _ORIG(*a)
    n = len(keys)
    return dq, keys, dk, np.tile(np.asarray(a[5], dtype=np.float64) / n, (n, 1))


@pytest.mark.parametrize("slip", [_without_D, _dq_unscaled, _dk_from_keys, _dv_uniform])
def test_planted_backward_slips_are_caught(monkeypatch, slip):
    monkeypatch.setattr(R, "attend_row_grad", slip)
    with pytest.raises(AssertionError):
        _check_finite_differences(n_probe=25)


# --- the saved-statistics form (p from lse, D from out) ------------------------------
def _saved_case(seed=5, seqlens=(37, 20), Hq=4, Hkv=2, d=8, B=8, topk=3):
    q, k, v, dout, cu = _case(list(seqlens), Hq, Hkv, d, seed)
    fw = R.forward(q, k, v, cu, Hq, Hkv, B, topk)
    return q, k, v, dout, cu, fw, (Hq, Hkv, B, topk)


def test_saved_statistics_form_equals_the_backward():
    """With the forward's exact out and lse, the saved-statistics backward is
    the pinned backward (which finite differences check)."""
    q, k, v, dout, cu, fw, (Hq, Hkv, B, topk) = _saved_case()
    ref = R.backward(q, k, v, cu, dout, Hq, Hkv, B, topk, idx=fw["idx"])
    got = R.backward_saved(q, k, v, cu, dout, fw["out"], fw["lse"], fw["idx"], Hq, Hkv, B, topk)
    for n in ("dq", "dk", "dv"):
        np.testing.assert_allclose(got[n], ref[n], rtol=0, atol=1e-10)
        assert np.all(got[n + "_abs"] >= np.abs(got[n]) - 1e-12)   # the budgets bound the results


def test_saved_statistics_slip_is_caught(monkeypatch):
    """A slip in the saved-statistics form (D from dout . v instead of dout .
    out) breaks the equality above."""
    orig = R.attend_row_grad_saved

    def slip(q_row, k_g, v_g, mask, scale, dout_row, lse_row, out_row):
        return orig(q_row, k_g, v_g, mask, scale, dout_row, lse_row, R.as_f64(v_g).mean(0))

    monkeypatch.setattr(R, "attend_row_grad_saved", slip)
    with pytest.raises(AssertionError):
        test_saved_statistics_form_equals_the_backward()


def test_sampled_form_equals_the_backward_at_every_row_and_key():
    """The sampled saved-statistics backward (a row's dq from its keys, a key's
    dk / dv summed over the rows that attend it) gives the pinned backward's
    dq, dk, dv and the full form's absolute-term sums at every row and key,
    including keys of short last blocks and keys no row attends."""
    q, k, v, dout, cu, fw, (Hq, Hkv, B, topk) = _saved_case()
    ref = R.backward(q, k, v, cu, dout, Hq, Hkv, B, topk, idx=fw["idx"])
    full = R.backward_saved(q, k, v, cu, dout, fw["out"], fw["lse"], fw["idx"], Hq, Hkv, B, topk)
    T = q.shape[0]
    rows = [(t, h) for t in range(T) for h in range(Hq)]
    keys = [(u, g) for u in range(T) for g in range(Hkv)]
    got = R.backward_saved_sample(q, k, v, cu, dout, fw["out"], fw["lse"], fw["idx"], Hq, Hkv,
                                  B, topk, rows=rows, keys=keys)
    ri = tuple(np.array(rows).T)
    ki = tuple(np.array(keys).T)
    np.testing.assert_allclose(got["dq"], ref["dq"][ri], rtol=0, atol=1e-10)
    np.testing.assert_allclose(got["dk"], ref["dk"][ki], rtol=0, atol=1e-10)
    np.testing.assert_allclose(got["dv"], ref["dv"][ki], rtol=0, atol=1e-10)
    for n, sel in (("dq_abs", ri), ("dk_abs", ki), ("dv_abs", ki)):
        np.testing.assert_allclose(got[n], full[n][sel], rtol=1e-12, atol=1e-12)


def test_sampled_form_reads_bf16_bit_patterns():
    """Given bf16 bit patterns (uint16) it reads the same values as given the
    floats they encode."""
    q, k, v, dout, cu, fw, (Hq, Hkv, B, topk) = _saved_case()
    tb = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16)
    bits = lambda a: tb(a).view(torch.int16).numpy().view(np.uint16)
    flt = lambda a: tb(a).double().numpy()
    rows, keys = [(3, 1), (40, 0)], [(0, 0), (21, 0)]
    a = R.backward_saved_sample(bits(q), bits(k), bits(v), cu, bits(dout), bits(fw["out"]),
                                fw["lse"], fw["idx"], Hq, Hkv, B, topk, rows=rows, keys=keys)
    b = R.backward_saved_sample(flt(q), flt(k), flt(v), cu, flt(dout), flt(fw["out"]),
                                fw["lse"], fw["idx"], Hq, Hkv, B, topk, rows=rows, keys=keys)
    for n in a:
        np.testing.assert_array_equal(a[n], b[n])
