"""Plant plausible mistakes in the CPU oracle and check that a pin catches each.

Every mutation below replaces one oracle function (CPU only, via monkeypatch)
with a version carrying a typical slip; the named pin must then fail.  This is
what shows that the pins constrain the oracle rather than restate it.
"""
import math

import numpy as np
import pytest

from oracle import moba_ref as R
from tests import test_oracle_pins as P


def _own_block_outside_k(scores, j, topk):
    if j + 1 <= topk + 1:
        return list(range(j + 1)), False
    order = sorted(range(j), key=lambda i: (-float(scores[i]), i))
    return sorted(order[:topk] + [j]), False


def _tie_to_higher_index(scores, j, topk):
    if j + 1 <= topk:
        return list(range(j + 1)), False
    order = sorted(range(j), key=lambda i: (-float(scores[i]), -i))
    return sorted(order[:topk - 1] + [j]), True


def _no_token_causal_mask(sel, t, L, B, keys=None):
    u = np.arange(L) if keys is None else np.asarray(keys)
    return np.isin(u // B, np.asarray(list(sel))) & (u // B <= t // B)


def _mean_off_by_one(k_seq, B):
    L = k_seq.shape[0]
    nfull = L // B
    out = np.empty((nfull,) + tuple(k_seq.shape[1:]))
    for i in range(nfull):
        out[i] = R.as_f64(k_seq[i * B:(i + 1) * B - 1]).mean(axis=0)
    return out


def _merge_without_weights(parts):
    parts = list(parts)
    o = sum(np.asarray(p[0]) for p in parts) / len(parts)
    return o, max(p[1] for p in parts)


def _values_are_keys(q_row, k_g, v_g, mask, scale):
    return _ORIG_ATTEND(q_row, k_g, k_g, mask, scale)


def _scale_one_over_d(d, scale):
    return 1.0 / d


def _past_blocks_any_order(scores, j, topk):
    # keeps the LAST topk-1 past blocks instead of the best-scoring ones
    if j + 1 <= topk:
        return list(range(j + 1)), False
    return list(range(j - topk + 1, j + 1)), False


_ORIG_ATTEND = R.attend_row

MUTATIONS = [
    ("select_blocks", _own_block_outside_k, [P.test_p5_sparsity_from_explicit_mask]),
    ("select_blocks", _tie_to_higher_index, [P.test_p4_exact_tie_prefers_lower_index]),
    ("select_blocks", _past_blocks_any_order, [P.test_p4_topk_matches_library_sort]),
    ("moba_mask_row", _no_token_causal_mask, [lambda: P.test_p2_seamless_switch_is_full_causal(1, 1)]),
    ("block_means", _mean_off_by_one, [lambda: P.test_p1_brute_force_matches_vectorised(P.TINY[1])]),
    ("lse_merge", _merge_without_weights, [P.test_p7_lse_merge_equals_one_shot]),
    ("attend_row", _values_are_keys, [lambda: P.test_p3_topk1_is_block_diagonal_causal()]),
    ("_default_scale", _scale_one_over_d, [lambda: P.test_p2_seamless_switch_is_full_causal(4, 2)]),
]


@pytest.mark.parametrize("name,fn,pins", MUTATIONS, ids=[f"{m[0]}:{m[1].__name__}" for m in MUTATIONS])
def test_pin_catches_mutation(monkeypatch, name, fn, pins):
    monkeypatch.setattr(R, name, fn)
    for pin in pins:
        with pytest.raises(AssertionError):
            pin()


def test_gqa_group_mapping_is_pinned(monkeypatch):
    """Routing head h to KV head h % Hkv (instead of h // G) breaks the GQA switch pin."""
    orig = R.forward_rows

    def wrong_group(q_rows, t_local, heads, k_seq, v_seq, n_heads, n_kv_heads, *a, **kw):
        G = n_heads // n_kv_heads
        remapped = [(h % n_kv_heads) * G for h in heads]
        return orig(q_rows, t_local, remapped, k_seq, v_seq, n_heads, n_kv_heads, *a, **kw)

    monkeypatch.setattr(R, "forward_rows", wrong_group)
    with pytest.raises(AssertionError):
        P.test_p2_seamless_switch_is_full_causal(4, 2)
