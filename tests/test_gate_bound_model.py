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
