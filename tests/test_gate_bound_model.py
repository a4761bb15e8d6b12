"""Model, in plain Python, of the gate's selection for rows with more than 256
past blocks (group-maxima bound, then an index-carrying insertion list), run
step for step as the kernel does and checked against the oracle's selection
(score descending, ties to the lower block index) on random, tie-heavy and
all-equal score rows.  CPU only: it checks the algorithm, the GPU parity tests
check the kernel."""
import numpy as np
import pytest

from oracle import moba_ref as R


def _pair_merge(a, hi, lo, K):
    inf = np.float32(np.inf)

    def A(i):
        return inf if i < 0 else a[i]
    return [max(A(p), min(A(p - 1), hi), min(A(p - 2), lo)) for p in range(K)]


def _bounded_select(sc, K):
    sc = np.asarray(sc, dtype=np.float32)
    j = len(sc)
    gm = [np.float32(-np.inf)] * 32          # pass 1: maxima of 32 interleaved groups
    for i in range(j):
        gm[i % 32] = max(gm[i % 32], sc[i])
    a = [np.float32(-np.inf)] * K
    for x in range(0, 32, 2):
        a = _pair_merge(a, max(gm[x], gm[x + 1]), min(gm[x], gm[x + 1]), K)
    tau0 = a[K - 1]
    av, ai = [np.float32(-np.inf)] * K, [2 ** 31 - 1] * K
    for base in range(0, j, 32):             # pass 2: 32-column loads in block order
        thr = av[K - 1]
        for x in range(32):
            i = base + x
            if i >= j or not (sc[i] >= tau0 and sc[i] > thr):
                continue
            v = sc[i]
            nav, nai = av[:], ai[:]
            for p in range(K - 1, 0, -1):
                if v > av[p - 1]:
                    nav[p], nai[p] = av[p - 1], ai[p - 1]
                elif v > av[p]:
                    nav[p], nai[p] = v, i
            if v > av[0]:
                nav[0], nai[0] = v, i
            av, ai = nav, nai
    return sorted(ai)


@pytest.mark.parametrize("kind", ["normal", "ties", "all_equal"])
def test_bounded_selection_equals_the_oracle(kind):
    rng = np.random.default_rng({"normal": 1, "ties": 2, "all_equal": 3}[kind])
    for _ in range(150):
        j = int(rng.integers(257, 2600))
        topk = int(rng.choice([2, 3, 5, 9, 12, 16]))
        if kind == "normal":
            sc = rng.standard_normal(j).astype(np.float32)
        elif kind == "ties":
            sc = rng.integers(0, 5, j).astype(np.float32)
        else:
            sc = np.full(j, 0.25, np.float32)
            sc[rng.integers(0, j, 4)] = 1.0
        ref, _ = R.select_blocks(sc.astype(np.float64), j, topk)   # past blocks then own block j
        assert _bounded_select(sc, topk - 1) + [j] == ref


def _threshold_select(sc, K):
    """The original pass 1 over every score (merge network), then pass 2
    over every score: the exact cut tau, winners above it, ties at tau to
    the lowest blocks, ascending."""
    a = [np.float32(-np.inf)] * K
    for x in range(0, len(sc), 2):
        v0 = sc[x]
        v1 = sc[x + 1] if x + 1 < len(sc) else np.float32(-np.inf)
        a = _pair_merge(a, max(v0, v1), min(v0, v1), K)
    return _emit(list(enumerate(sc)), a, K)


def _emit(cands, a, K):
    tau = a[K - 1]
    need_eq = K - sum(1 for v in a if v > tau)
    out = []
    for i, v in cands:                          # block order
        take = v > tau or (v == tau and need_eq > 0)
        if take and not v > tau:
            need_eq -= 1
        if take and len(out) < K:
            out.append(i)
    return out


KCAND = 24


def _list_select(sc, K):
    """Rows with at most 256 past blocks: group-maxima bound tau0, the scores
    >= tau0 with their blocks into a list of KCAND (in block order), the cut
    and the winners over the list; a row whose list overflows takes both
    passes over every score instead."""
    sc = np.asarray(sc, dtype=np.float32)
    j = len(sc)
    gm = [np.float32(-np.inf)] * 32
    for i in range(j):
        gm[i % 32] = max(gm[i % 32], sc[i])
    g = [np.float32(-np.inf)] * K
    for x in range(0, 32, 2):
        g = _pair_merge(g, max(gm[x], gm[x + 1]), min(gm[x], gm[x + 1]), K)
    tau0 = g[K - 1]
    cands = [(i, sc[i]) for i in range(j) if sc[i] >= tau0]
    if len(cands) > KCAND:
        return _threshold_select(sc, K), True
    a = [np.float32(-np.inf)] * K
    for x in range(0, len(cands), 2):
        v0 = cands[x][1]
        v1 = cands[x + 1][1] if x + 1 < len(cands) else np.float32(-np.inf)
        a = _pair_merge(a, max(v0, v1), min(v0, v1), K)
    return _emit(cands, a, K), False


@pytest.mark.parametrize("kind", ["normal", "ties", "all_equal", "near_ties"])
def test_list_selection_equals_the_oracle(kind):
    rng = np.random.default_rng({"normal": 11, "ties": 12, "all_equal": 13, "near_ties": 14}[kind])
    fallbacks = 0
    for _ in range(300):
        topk = int(rng.choice([2, 3, 5, 9, 12, 16]))
        j = int(rng.integers(topk, 257))      # rows scored on the tensor cores: j + 1 > topk
        if kind == "normal":
            sc = rng.standard_normal(j).astype(np.float32)
        elif kind == "ties":
            sc = rng.integers(0, 5, j).astype(np.float32)
        elif kind == "all_equal":
            sc = np.full(j, 0.25, np.float32)
            sc[rng.integers(0, j, 4)] = 1.0
        else:                                  # bit-identical copies on and around the cut
            sc = rng.standard_normal(j).astype(np.float32)
            sc[rng.integers(0, j, 6)] = sc[int(rng.integers(0, j))]
        got, fell_back = _list_select(sc, topk - 1)
        fallbacks += fell_back
        ref, _ = R.select_blocks(sc.astype(np.float64), j, topk)
        assert got + [j] == ref
    if kind == "normal":
        assert fallbacks == 0                  # random rows fit the list
    if kind == "all_equal":
        assert fallbacks > 0                   # and the fallback is exercised
