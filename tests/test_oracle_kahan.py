"""Pins of the oracle's Kahan-compensated SGD step (bf16 parameters, bf16
compensation, bf16 gradient): a hand-worked sequence, dyadic closed forms,
special cases, and the accumulation bound of compensated summation against
float64 sums (where plain bf16 SGD stalls)."""
import numpy as np
import pytest
import torch


def bits(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def vals(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def test_hand_worked_sequence(orc):
    """p = 1, c = 0, g = 1, lr = 2^-10: u = -2^-10 is a quarter of the bf16
    spacing just below 1 (2^-8).  Step by step (round to nearest, ties to even):
      1: 1 - 2^-10     -> p = 1,          c = -2^-10
      2: 1 - 2^-9      -> tie, p = 1 (even), c = -2^-9
      3: 1 - 3 * 2^-10 -> p = 1 - 2^-8,   c = -3*2^-10 + 2^-8 = 2^-10
      4: y = 0         -> p = 1 - 2^-8,   c = 0
    so after four steps p is exactly 1 - 4 * 2^-10, where plain bf16 SGD would
    have stayed at 1."""
    p, c, g = bits([1.0]), bits([0.0]), bits([1.0])
    want = [(1.0, -2.0**-10), (1.0, -2.0**-9), (1.0 - 2.0**-8, 2.0**-10), (1.0 - 2.0**-8, 0.0)]
    for wp, wc in want:
        p, c = orc.kahan_sgd(p, c, g, 2.0**-10)
        assert vals(p)[0] == wp and vals(c)[0] == wc


def test_dyadic_exact_step(orc):
    """Every operation exact and p + y on the bf16 grid: p' = p - lr g, c' = 0."""
    rng = np.random.default_rng(0)
    p0 = rng.integers(-64, 64, 1000).astype(np.float32) / 8          # multiples of 1/8 in [-8, 8)
    g0 = rng.integers(-16, 16, 1000).astype(np.float32)               # integers
    lr = 2.0**-3
    p, c = orc.kahan_sgd(bits(p0), bits(np.zeros(1000)), bits(g0), lr)
    assert np.array_equal(vals(p), p0 - lr * g0)
    assert np.all(vals(c) == 0)


def test_special_cases(orc):
    rng = np.random.default_rng(1)
    p0 = bits(rng.standard_normal(500))
    c0 = bits(rng.standard_normal(500) * 2.0**-12)
    g0 = bits(rng.standard_normal(500))
    # lr = 0 and no compensation: nothing moves
    p, c = orc.kahan_sgd(p0, bits(np.zeros(500)), g0, 0.0)
    assert np.array_equal(p, p0) and np.all(vals(c) == 0)
    # zero gradient: the stored compensation is applied as far as the grid allows
    p, c = orc.kahan_sgd(p0, c0, bits(np.zeros(500)), 0.1)
    pv, cv = vals(p0).astype(np.float64), vals(c0).astype(np.float64)
    assert np.array_equal(p, bits(pv + cv))                          # one rounding of an exact sum
    assert np.array_equal(vals(c), vals(bits(cv - (vals(p).astype(np.float64) - pv))))
    # NaN parameters stay NaN
    p, _ = orc.kahan_sgd(bits([np.nan, 1.0]), bits([0.0, 0.0]), bits([1.0, np.nan]), 0.5)
    assert np.all(np.isnan(vals(p)))


@pytest.mark.parametrize("scale", [1.0, 1e3])
def test_compensated_accumulation_bound(orc, scale):
    """N steps with increments far below half a bf16 spacing of p: plain bf16
    SGD stalls (each increment rounds away), compensated SGD tracks the exact
    sum.  Per step the only uncompensated error is the rounding of c' to bf16
    (at most 2^-9 |c'|, |c'| at most half a spacing of p plus |u|) and of the
    fp32 sum y (2^-24 |y|), so |p_N + c_N - (p_0 + sum u)| <=
    N (2^-9 (s/2 + |u|max) + 2^-24 (s + |u|max)), s the largest spacing of p met."""
    rng = np.random.default_rng(2)
    n, N, lr = 256, 1500, 1e-4
    p0 = bits(scale * (1.0 + rng.random(n)))
    p, c = p0.copy(), bits(np.zeros(n))
    plain = vals(p0).copy()
    exact = vals(p0).astype(np.float64)
    umax = 0.0
    for _ in range(N):
        g = bits(scale * (1.0 + 0.5 * rng.standard_normal(n)))       # biased: the sum drifts steadily
        u = -(np.float32(lr) * vals(g))                                # the fp32 increments, as the step forms them
        exact += u.astype(np.float64)
        umax = max(umax, float(np.abs(u).max()))
        plain = vals(bits(plain + u))                                  # plain bf16 SGD
        p, c = orc.kahan_sgd(p, c, g, lr)
    got = vals(p).astype(np.float64) + vals(c).astype(np.float64)
    s = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(vals(p0)), np.abs(vals(p))))) - 7)
    bound = N * (2.0**-9 * (s / 2 + umax) + 2.0**-24 * (s + umax))
    assert np.all(np.abs(got - exact) <= bound)
    drift = np.abs(exact - vals(p0))
    assert np.all(np.abs(plain - exact) > 0.5 * drift)                 # plain SGD lost most of the drift
    assert np.median(np.abs(got - exact)) < 0.02 * np.median(drift)    # compensated SGD kept it
