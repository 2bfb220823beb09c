"""The parity checker itself, on the CPU: the oracle stands in for both sides,
and mistakes are planted on the oracle's side, so that the checks the GPU
tests rely on are shown to pass on a correct step and to fail on a wrong one."""
import numpy as np
import pytest

from synthetic import make_labels, make_W_f32, make_X, workload
from tests.parity import (check_step, flip_corrected_weights, operand_codes, operand_of_logit, operand_format,
                          positives)


def _step(orc, dtype, L=300, d=64, B=12, seed=1, step=2):
    w = workload("tiny", dtype="fp8" if dtype != "bf16" else "bf16", L=L, d=d, B=B)
    wd = {"bf16": "bf16", "fp8": "fp8", "e5m2": "e5m2"}[dtype]
    W = orc.sr_round(make_W_f32(w, std=0.002), wd, 0, 2**64 - 1)
    X = make_X(w, step)
    rowptr, cols = make_labels(w, step)
    r = orc.train_step(W, X, rowptr, cols, w.lr, seed, step, dtype, want_zg=True)
    return w, W, X, rowptr, cols, r


def _neighbour_operand(g, dtype):
    """G moved one grid step away from zero (as a differing rounding of the
    same logit would put it)."""
    import ml_dtypes
    fmt = operand_format(dtype)
    if fmt == "bf16":
        c = np.float32(g).astype(ml_dtypes.bfloat16).view(np.uint16) + np.uint16(1)
        return float(c.view(ml_dtypes.bfloat16).astype(np.float64))
    t = ml_dtypes.float8_e4m3fn if fmt == "e4m3" else ml_dtypes.float8_e5m2
    c = (np.float32(g) * np.float32(256)).astype(t).view(np.uint8) + np.uint8(1)
    return float(c.view(t).astype(np.float64)) / 256.0


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "e5m2"])
def test_oracle_against_itself_passes(orc, dtype):
    w, W, X, rowptr, cols, r = _step(orc, dtype)
    _, flips = check_step(orc, W, X, rowptr, cols, w.lr, 1, 2, dtype, r["W"], r["dX"], r["Z"], r["G"])
    assert flips == 0


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "e5m2"])
def test_restep_without_flips_is_the_oracle(orc, dtype):
    w, W, X, rowptr, cols, r = _step(orc, dtype)
    out, rows = flip_corrected_weights(orc, W, X, r["G"], r["G"], r["W"], w.lr, 1, 2, dtype)
    assert rows == 0 and np.array_equal(out, r["W"])


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "e5m2"])
def test_one_flip_restep_moves_only_its_row(orc, dtype):
    """A positive's operand (|G| near 1/2, the largest a flip can move) one
    grid step away: every row but that label's keeps the oracle's codes, and
    that row is re-stepped (the internal check reproduces the oracle's codes
    from the oracle's operands first)."""
    w, W, X, rowptr, cols, r = _step(orc, dtype)
    Y = positives(rowptr, cols, w.L, w.B)
    l, b = map(int, np.argwhere(Y > 0)[0])
    Gf = r["G"].copy()
    Gf[l, b] = _neighbour_operand(Gf[l, b], dtype)
    assert abs(int(operand_codes(Gf, dtype)[l, b]) - int(operand_codes(r["G"], dtype)[l, b])) == 1
    out, rows = flip_corrected_weights(orc, W, X, Gf, r["G"], r["W"], w.lr, 1, 2, dtype)
    assert rows == 1
    others = np.ones(w.L, bool)
    others[l] = False
    assert np.array_equal(out[others], r["W"][others])
    assert not np.array_equal(out[l], r["W"][l])


def test_planted_mistakes_fail(orc):
    """Wrong operands, a wrong dX term and biased weights each fail the check."""
    dtype = "bf16"
    w, W, X, rowptr, cols, r = _step(orc, dtype)
    args = (orc, W, X, rowptr, cols, w.lr, 1, 2, dtype)
    # an operand that is not the rounded operand of its own logit
    Gbad = r["G"].copy()
    Gbad[3, 4] += 0.25
    with pytest.raises(AssertionError):
        check_step(*args, r["W"], r["dX"], r["Z"], Gbad)
    # a dX row with one label's term counted twice
    dXbad = r["dX"].copy()
    dXbad[2] += r["G"][7, 2] * orc.w_value(W[7], "bf16")
    with pytest.raises(AssertionError, match="dX"):
        check_step(*args, r["W"], dXbad, r["Z"], r["G"])
    # weights rounded down one step too often: a signed bias
    Wbad = r["W"].copy()
    part = Wbad[: w.L // 4]
    neg = (part & 0x8000) != 0
    part[:] = np.where(neg, part + 1, np.where(part == 0, 0x8001, part - 1))   # one step toward -inf
    with pytest.raises(AssertionError, match="mean signed error"):
        check_step(*args, Wbad, r["dX"], r["Z"], r["G"])


def test_operand_of_logit_pins(orc):
    """The checker's operand of a logit at values fixed by the definition:
    sigmoid(0) = 1/2 exactly; sigmoid(-30) rounds to a tiny positive value;
    a positive at z = 0 gives -1/2."""
    z = np.array([[0.0, 0.0, -30.0]], np.float32)
    y = np.array([[0.0, 1.0, 0.0]], np.float32)
    g = operand_of_logit(z, y, "bf16")
    assert g[0, 0] == 0.5 and g[0, 1] == -0.5 and 0 < g[0, 2] < 1e-12
    g8 = operand_of_logit(z, y, "e4m3")
    assert g8[0, 0] == 0.5 and g8[0, 1] == -0.5 and g8[0, 2] == 0.0


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "fp8_ge5m2"])
def test_oracle_operands_next_to_midpoints(orc, dtype):
    """The oracle's gradient operands at logits built next to the operand
    grid's rounding midpoints (the construction of the GPU midpoint test)
    equal sigmoid in double rounded to fp32, then to the grid (numpy and
    ml_dtypes); about a fifth of these logits have an fp32 neighbour that
    rounds to another operand."""
    import ml_dtypes
    from tests.test_gpu_operand_midpoints import _layout, _midpoint_logits, _parts
    fmt = operand_format(dtype)
    P, scales, wgrid, lr, B = _layout(dtype)
    d, L = 768, 128
    rng = np.random.default_rng(7)
    Y = np.zeros((L, B), np.float32)
    for b in range(B):
        Y[b % L, b] = 1.0
    target = np.where(Y > 0, rng.choice(_midpoint_logits(fmt, 1), size=(L, B)),
                      rng.choice(_midpoint_logits(fmt, 0), size=(L, B))).astype(np.float32)
    parts, _ = _parts(target, wgrid, scales)
    X = np.zeros((B, d), np.float32)
    W = np.zeros((L, d), np.float64)
    for b in range(B):
        for j in range(P):
            X[b, b * P + j] = scales[j]
            W[:, b * P + j] = parts[j][:, b].astype(np.float64)
    Xb = X.astype(ml_dtypes.bfloat16).view(np.uint16)
    Wc = W.astype(wgrid).view(np.uint16 if dtype == "bf16" else np.uint8)
    cols = np.concatenate([np.nonzero(Y[:, b])[0] for b in range(B)]).astype(np.int32)
    rowptr = np.concatenate([[0], np.cumsum((Y > 0).sum(axis=0))]).astype(np.int32)
    r = orc.train_step(Wc, Xb, rowptr, cols, 0.0, 0, 0, dtype, want_zg=True, want_dx=False)
    assert np.mean(r["Z"] == target) > 0.99
    want = operand_of_logit(r["Z"], Y, fmt)
    assert np.array_equal(r["G"], want)
    up = operand_of_logit(np.nextafter(r["Z"], np.float32(np.inf)), Y, fmt)
    assert np.mean(up != want) > 0.05
