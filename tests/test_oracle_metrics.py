"""Pins of the oracle's P@k: a worked example computed by hand, brute force
with Python sets on random data, and the closed forms of perfect and
hopeless predictions."""
import numpy as np
import pytest


def test_precision_at_k_worked_example(orc):
    # row 0 predicts 5, 7, 9 with positives {7, 9, 11}: hits 0, 1, 2 in the first 1, 2, 3
    # row 1 predicts 1, 2, 3 with positives {1}:        hits 1, 1, 1
    # P@1 = (0/1 + 1/1)/2, P@2 = (1/2 + 1/2)/2, P@3 = (2/3 + 1/3)/2
    idx = np.array([[5, 7, 9], [1, 2, 3]], np.int32)
    rowptr = np.array([0, 3, 4], np.int32)
    cols = np.array([7, 9, 11, 1], np.int32)
    assert orc.precision_at_k(idx, rowptr, cols).tolist() == [0.5, 0.5, 0.5]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_precision_at_k_brute_force(orc, seed):
    rng = np.random.default_rng(seed)
    B, k, L = 37, 9, 60
    idx = np.stack([rng.permutation(L)[:k] for _ in range(B)]).astype(np.int32)
    sets = [set(rng.choice(L, size=rng.integers(0, 12), replace=False).tolist()) for _ in range(B)]
    rowptr = np.cumsum([0] + [len(s) for s in sets]).astype(np.int32)
    cols = np.array([c for s in sets for c in sorted(s)], np.int32)
    want = [np.mean([len(set(idx[b, :j].tolist()) & sets[b]) / j for b in range(B)]) for j in range(1, k + 1)]
    assert np.allclose(orc.precision_at_k(idx, rowptr, cols), want, rtol=0, atol=1e-15)


def test_precision_at_k_closed_forms(orc):
    B, k = 5, 4
    pos = [[3, 8], [1], [2, 4, 6, 7, 9], [], [0, 5, 10]]
    rowptr = np.cumsum([0] + [len(p) for p in pos]).astype(np.int32)
    cols = np.array([c for p in pos for c in p], np.int32)
    # perfect: positives first, then labels that are not positives -> P@j = mean(min(|Y|, j) / j)
    idx = np.array([(p + [100 + i for i in range(k)])[:k] for p in pos], np.int32)
    want = [np.mean([min(len(p), j) / j for p in pos]) for j in range(1, k + 1)]
    assert np.allclose(orc.precision_at_k(idx, rowptr, cols), want, rtol=0, atol=1e-15)
    # hopeless: no prediction is a positive
    none = np.full((B, k), 1000, np.int32) + np.arange(k, dtype=np.int32)
    assert orc.precision_at_k(none, rowptr, cols).tolist() == [0.0] * k
