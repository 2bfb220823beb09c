"""Pins of the oracle's top-k: brute-force sort on exactly representable
scores (with forced ties), float64 consistency on random data, NaN order."""
import ml_dtypes
import numpy as np
import pytest

from synthetic import bf16_bits, bf16_value


def _brute(scores, k):
    # rank: score descending, ties by lower index (np.lexsort: last key primary)
    idx = np.arange(scores.size)
    order = np.lexsort((idx, -scores))
    return order[:k]


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "e5m2"])
def test_topk_exact_ties_lower_index(orc, dtype):
    rng = np.random.default_rng(20)
    B, d, L, k = 5, 32, 200, 7
    xv = (rng.integers(-4, 5, (B, d)) / 4).astype(np.float32)
    wv = (rng.integers(-4, 5, (L, d)) / 32).astype(np.float32)
    wv[150] = wv[10]; wv[151] = wv[10]; wv[3] = wv[199]       # exact ties
    X = bf16_bits(xv)
    fmt = ml_dtypes.float8_e5m2 if dtype == "e5m2" else ml_dtypes.float8_e4m3fn     # k/32, |k| <= 4: on both grids
    W = bf16_bits(wv) if dtype == "bf16" else wv.astype(fmt).view(np.uint8)
    idx, sc = orc.topk(W, X, k, dtype, nthreads=3)
    S = xv.astype(np.float64) @ wv.astype(np.float64).T      # exact
    for b in range(B):
        ref = _brute(S[b], k)
        assert idx[b].tolist() == ref.tolist()
        assert np.array_equal(sc[b], S[b, ref].astype(np.float32))
    # rows where the tie is inside the top-k list the lower index first
    for b in range(B):
        if 10 in idx[b] and 150 in idx[b]:
            assert idx[b].tolist().index(10) < idx[b].tolist().index(150)


def test_topk_random_consistent_with_float64(orc):
    rng = np.random.default_rng(21)
    B, d, L, k = 4, 64, 1000, 5
    X = bf16_bits((rng.standard_normal((B, d)) / 8).astype(np.float32))
    W = (rng.standard_normal((L, d)) * 0.02).astype(np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    idx, sc = orc.topk(W, X, k, "fp8", rows=[3, 1], nthreads=2)
    S = bf16_value(X).astype(np.float64) @ orc.e4m3_value(W).astype(np.float64).T
    for r, b in enumerate([3, 1]):
        ref = _brute(S[b], k)
        assert idx[r].tolist() == ref.tolist()          # no near-ties at this size
        for q in range(k):
            assert sc[r, q] == orc.score(W, X, int(idx[r, q]), b, "fp8")
        assert np.all(np.diff(sc[r]) <= 0)


def test_topk_nan_ranks_last(orc):
    rng = np.random.default_rng(22)
    B, d, L = 2, 16, 12
    X = bf16_bits(rng.standard_normal((B, d)).astype(np.float32))
    W = (rng.standard_normal((L, d)) * 0.1).astype(np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    W[[0, 4, 5]] = 0x7F                                   # NaN rows
    idx, sc = orc.topk(W, X, L, "fp8")
    for b in range(B):
        assert idx[b, -3:].tolist() == [0, 4, 5]
        assert np.all(np.isnan(sc[b, -3:])) and not np.any(np.isnan(sc[b, :-3]))
