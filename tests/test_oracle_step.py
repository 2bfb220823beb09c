"""Pins of the oracle's training step: exact dyadic cases against float64
brute force composed from library routines, a finite-difference check of the
gradient, special cases with closed forms, invariances and error paths."""
import ml_dtypes
import numpy as np
import pytest
import torch
from scipy.special import expit

from synthetic import bf16_bits, bf16_value, labels_dense


def _csr(rows):
    rowptr = np.zeros(len(rows) + 1, np.int32)
    rowptr[1:] = np.cumsum([len(r) for r in rows])
    cols = np.array([c for r in rows for c in r], np.int32)
    return rowptr, cols


def _rne_bf16_val(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def _rne_e4m3_val(x):
    return np.asarray(x, np.float32).astype(ml_dtypes.float8_e4m3fn).astype(np.float32)


def _rne_e5m2_val(x):
    return np.asarray(x, np.float32).astype(ml_dtypes.float8_e5m2).astype(np.float32)


def _w_codes(wf, dtype):
    """Weights on the head's grid (RNE): bf16 bits, E4M3 or E5M2 codes."""
    if dtype == "bf16":
        return bf16_bits(wf)
    fmt = ml_dtypes.float8_e5m2 if dtype == "e5m2" else ml_dtypes.float8_e4m3fn
    return np.asarray(wf, np.float32).astype(fmt).view(np.uint8)


def _dyadic_case(rng, B, d, L, dtype):
    # X: integers in [-8, 8] / 8; W: integers in [-8, 8] / 64 (exact in both
    # grids); every sum below is exact in fp32.
    xv = (rng.integers(-8, 9, (B, d)) / 8).astype(np.float32)
    wv = (rng.integers(-8, 9, (L, d)) / 64).astype(np.float32)
    X = bf16_bits(xv)
    W = _w_codes(wv, dtype)
    rows = [sorted(set(rng.integers(0, L, 1 + int(rng.integers(0, 4))).tolist())) for _ in range(B)]
    return X, W, xv, wv, _csr(rows)


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "fp8_ge5m2", "e5m2"])
def test_step_exact_dyadic_case(orc, dtype):
    rng = np.random.default_rng(10)
    B, d, L = 6, 16, 40
    X, W, xv, wv, (rowptr, cols) = _dyadic_case(rng, B, d, L, dtype)
    lr, seed, step = 0.5, 42, 3
    r = orc.train_step(W, X, rowptr, cols, lr, seed, step, dtype, want_zg=True, nthreads=3)
    Y = labels_dense(rowptr, cols, L)                       # [B, L]
    Z64 = xv.astype(np.float64) @ wv.astype(np.float64).T   # [B, L], exact
    assert np.array_equal(r["Z"], Z64.T.astype(np.float32))
    g = expit(Z64).astype(np.float32) - Y                   # fp32 sigmoid minus y
    if dtype == "bf16":
        Gh = _rne_bf16_val(g)
    elif dtype in ("fp8", "e5m2"):                          # E4M3 gradient operand (E5M2 heads too)
        Gh = _rne_e4m3_val(g * np.float32(256)) / np.float32(256)
    else:                                                   # E5M2 gradient operand, same 2^8 scale
        Gh = _rne_e5m2_val(g * np.float32(256)) / np.float32(256)
    assert np.array_equal(r["G"], Gh.T)
    dw = Gh.T.astype(np.float64) @ xv.astype(np.float64)    # [L, d], exact
    v = (wv - (np.float32(lr) * dw.astype(np.float32))).astype(np.float32)
    k = orc.draw16(seed, step, 0, L * d).reshape(L, d)
    expect_W = orc.sr_with_draws(v, k, dtype).reshape(L, d)
    assert np.array_equal(r["W"], expect_W)
    dX = Gh.astype(np.float64) @ wv.astype(np.float64)      # [B, d], exact
    assert np.array_equal(r["dX"], dX.astype(np.float32))


def _random_case(w_dtype, B=8, d=48, L=300, seed=0):
    rng = np.random.default_rng(seed)
    X = bf16_bits((rng.standard_normal((B, d)) / np.sqrt(d)).astype(np.float32))
    wf = (rng.standard_normal((L, d)) * 0.3).astype(np.float32)
    W = _w_codes(wf, "e5m2" if w_dtype == "e5m2" else ("bf16" if w_dtype == "bf16" else "fp8"))
    rows = [rng.integers(0, L, 1 + int(rng.integers(0, 5))).tolist() for _ in range(B)]
    return X, W, _csr(rows)


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "fp8_ge5m2", "e5m2"])
def test_step_random_case_within_fp32_bounds(orc, dtype):
    X, W, (rowptr, cols) = _random_case(dtype)
    L, d = W.shape
    B = X.shape[0]
    r = orc.train_step(W, X, rowptr, cols, 0.05, 1, 2, dtype, want_zg=True)
    wv = orc.w_value(W, dtype).reshape(L, d).astype(np.float64)
    if dtype == "bf16":
        xq = bf16_value(X).astype(np.float64)
        sx = 1.0
    else:
        sx = orc.fp8_x_scale(X)
        xq = _rne_e4m3_val(bf16_value(X) * np.float32(sx)).astype(np.float64)
    Z64 = (xq @ wv.T) / sx
    bound = d * 2.0 ** -24 * (np.abs(xq) @ np.abs(wv).T) / sx + 1e-30
    assert np.all(np.abs(r["Z"].T - Z64) <= bound)
    # gradient operand: within one operand ulp of sigmoid(z) - y in float64
    Y = labels_dense(rowptr, cols, L)
    g64 = expit(Z64) - Y
    G = r["G"].T.astype(np.float64)
    if dtype == "bf16":
        assert np.all(np.abs(G - g64) <= 2.0 ** -8 * np.abs(g64) + 1e-6)
    elif dtype in ("fp8", "e5m2"):
        assert np.all(np.abs(G - g64) <= 2.0 ** -4 * np.abs(g64) + 2.0 ** -17 + 1e-6)
    else:       # E5M2 of 2^8 g: half a spacing is 2^-3 relative, subnormal spacing 2^-16 / 2^8
        assert np.all(np.abs(G - g64) <= 2.0 ** -3 * np.abs(g64) + 2.0 ** -25 + 1e-6)
    # dX = G W (old W), float64 brute force on the oracle's own operand values
    dX64 = G @ wv
    err_bound = L * 2.0 ** -24 * (np.abs(G) @ np.abs(wv)) + 1e-30
    assert np.all(np.abs(r["dX"] - dX64) <= err_bound)
    # updated weights: neighbours of v = w - lr * (G^T x) evaluated in float64
    xv = xq / sx
    v64 = wv - 0.05 * (G.T @ xv)
    new = orc.w_value(r["W"], dtype).reshape(L, d).astype(np.float64)
    if dtype == "bf16":
        grid = np.unique(np.arange(0, 0x7F80, dtype=np.uint16).view(ml_dtypes.bfloat16).astype(np.float64))
    elif dtype == "e5m2":
        grid = np.unique(np.arange(0, 0x7C, dtype=np.uint8).view(ml_dtypes.float8_e5m2).astype(np.float64))
    else:
        grid = np.unique(np.arange(0, 127, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64))
    a = np.abs(v64)
    i = np.searchsorted(grid, a, side="right") - 1
    lo = grid[np.clip(i - 1, 0, grid.size - 1)]
    hi = grid[np.clip(i + 2, 0, grid.size - 1)]           # one extra neighbour: v64 vs fp32 v
    assert np.all((np.abs(new) >= lo) & (np.abs(new) <= hi))


def test_gradient_matches_finite_difference_of_bce(orc):
    # l(z) = softplus(z) - y z  =>  dl/dz = sigmoid(z) - y
    X, W, (rowptr, cols) = _random_case("bf16", seed=3)
    L = W.shape[0]
    r = orc.train_step(W, X, rowptr, cols, 0.0, 0, 0, "bf16", want_zg=True)
    z = r["Z"].astype(np.float64)
    Y = labels_dense(rowptr, cols, L).T
    h = 1e-5
    loss = lambda t: np.logaddexp(0.0, t) - Y * t
    fd = (loss(z + h) - loss(z - h)) / (2 * h)
    assert np.all(np.abs(r["G"] - fd) <= 2.0 ** -8 * np.abs(fd) + 1e-7)
    assert np.all(r["G"][Y == 1] < 0) and np.all(r["G"][Y == 0] > 0)


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "fp8_ge5m2", "e5m2"])
def test_special_cases(orc, dtype):
    X, W, (rowptr, cols) = _random_case(dtype, seed=4)
    L, d = W.shape
    Y = labels_dense(rowptr, cols, L).T
    # W = 0: G = 1/2 - Y exactly and dX = 0
    r = orc.train_step(np.zeros_like(W), X, rowptr, cols, 0.1, 0, 0, dtype, want_zg=True)
    assert np.array_equal(r["G"], 0.5 - Y)
    assert np.all(r["dX"] == 0)
    # lr = 0: weights unchanged (as values: IEEE gives -0 - (-0) = +0)
    val = lambda a: orc.w_value(a, dtype)
    r = orc.train_step(W, X, rowptr, cols, 0.0, 5, 6, dtype)
    assert np.array_equal(val(r["W"]), val(W))
    # X = 0: dW = 0 so W is unchanged; G = 1/2 - Y
    r = orc.train_step(W, np.zeros_like(X), rowptr, cols, 0.3, 5, 6, dtype, want_zg=True)
    assert np.array_equal(val(r["W"]), val(W))
    assert np.array_equal(r["G"], 0.5 - Y)


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "fp8_ge5m2", "e5m2"])
def test_label_range_split_and_dx_rows(orc, dtype):
    X, W, (rowptr, cols) = _random_case(dtype, seed=5)
    L, d = W.shape
    full = orc.train_step(W, X, rowptr, cols, 0.05, 7, 8, dtype, want_zg=True, nthreads=4)
    a = orc.train_step(W, X, rowptr, cols, 0.05, 7, 8, dtype, l0=0, l1=123, want_zg=True, nthreads=1)
    b = orc.train_step(W, X, rowptr, cols, 0.05, 7, 8, dtype, l0=123, l1=L, want_zg=True, nthreads=2)
    assert np.array_equal(np.concatenate([a["W"], b["W"]]), full["W"])
    assert np.array_equal(np.concatenate([a["Z"], b["Z"]]), full["Z"])
    assert np.array_equal(np.concatenate([a["G"], b["G"]]), full["G"])
    assert np.allclose(a["dX"] + b["dX"], full["dX"], rtol=1e-5, atol=1e-6)
    rows = orc.dx_rows(W, X, rowptr, cols, [0, 3, 7], dtype, nthreads=3)
    assert np.allclose(rows, full["dX"][[0, 3, 7]], rtol=1e-5, atol=1e-6)


def test_duplicate_positives_count_once_and_unsorted_rows(orc):
    X, W, _ = _random_case("bf16", seed=6)
    rows = [[5, 9], [1], [7, 3], [0], [2], [8], [4], [6]]
    dup = [[9, 5, 9, 5], [1, 1], [3, 7], [0], [2, 2, 2], [8], [4], [6]]
    r1 = orc.train_step(W, X, *_csr(rows), 0.05, 1, 1, "bf16", want_zg=True)
    r2 = orc.train_step(W, X, *_csr(dup), 0.05, 1, 1, "bf16", want_zg=True)
    assert np.array_equal(r1["G"], r2["G"]) and np.array_equal(r1["W"], r2["W"])


def test_fp8_x_scale_is_undone(orc):
    # doubling X leaves the E4M3 codes of x * s_X unchanged and halves s_X,
    # so the logits double exactly
    X, W, (rowptr, cols) = _random_case("fp8", seed=7)
    X2 = bf16_bits(bf16_value(X) * np.float32(2))
    r1 = orc.train_step(W, X, rowptr, cols, 0.0, 0, 0, "fp8", want_zg=True)
    r2 = orc.train_step(W, X2, rowptr, cols, 0.0, 0, 0, "fp8", want_zg=True)
    assert np.array_equal(r2["Z"], 2 * r1["Z"])


def test_malformed_csr_is_rejected(orc):
    X, W, (rowptr, cols) = _random_case("bf16", seed=8)
    L = W.shape[0]
    bad_cols = cols.copy(); bad_cols[0] = L
    with pytest.raises(orc.OracleError):
        orc.train_step(W, X, rowptr, bad_cols, 0.1, 0, 0, "bf16")
    bad_cols[0] = -1
    with pytest.raises(orc.OracleError):
        orc.train_step(W, X, rowptr, bad_cols, 0.1, 0, 0, "bf16")
    bad_ptr = rowptr.copy(); bad_ptr[2], bad_ptr[3] = bad_ptr[3], bad_ptr[2] - 1
    with pytest.raises(orc.OracleError):
        orc.train_step(W, X, bad_ptr, cols, 0.1, 0, 0, "bf16")
