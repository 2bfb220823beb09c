"""Pins of the oracle's stochastic rounding: grid fixed points, neighbours
from an independent enumeration of the grid, the closed-form probability of
rounding up, unbiasedness and the special values."""
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest


def _grid(dtype):
    """Sorted finite non-negative grid values, enumerated with ml_dtypes."""
    if dtype == "bf16":
        v = np.arange(0, 0x7F80, dtype=np.uint16).view(ml_dtypes.bfloat16).astype(np.float64)
    elif dtype == "e5m2":
        v = np.arange(0, 0x7C, dtype=np.uint8).view(ml_dtypes.float8_e5m2).astype(np.float64)
    else:
        v = np.arange(0, 127, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    return np.unique(v)


def _code_value(codes, dtype):
    if dtype == "bf16":
        return codes.view(ml_dtypes.bfloat16).astype(np.float64)
    if dtype == "e5m2":
        return codes.view(ml_dtypes.float8_e5m2).astype(np.float64)
    return codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "e5m2"])
def test_grid_points_are_fixed(orc, dtype):
    g = _grid(dtype)
    x = np.concatenate([g, -g]).astype(np.float32)
    rng = np.random.default_rng(3)
    k = rng.integers(0, 65536, x.size).astype(np.uint32)
    out = orc.sr_with_draws(x, k, dtype)
    assert np.array_equal(_code_value(out, dtype), x.astype(np.float64))
    # the sign of zero survives
    z = orc.sr_with_draws(np.array([-0.0, 0.0], np.float32), np.array([0, 65535], np.uint32), dtype)
    assert np.signbit(_code_value(z, dtype)).tolist() == [True, False]


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "e5m2"])
def test_result_is_a_neighbour(orc, dtype):
    g = _grid(dtype)
    rng = np.random.default_rng(4)
    top = {"fp8": 448.0, "e5m2": 57344.0, "bf16": 1e30}[dtype]
    lo_e = {"fp8": -12, "e5m2": -19, "bf16": -130}[dtype]
    x = (rng.random(30000) + 1) * np.exp2(rng.integers(lo_e, int(np.log2(top)), 30000))
    x = np.minimum(x, top * 0.999).astype(np.float32)
    x = np.where(rng.random(x.size) < 0.5, -x, x).astype(np.float32)
    k = rng.integers(0, 65536, x.size).astype(np.uint32)
    out = _code_value(orc.sr_with_draws(x, k, dtype), dtype)
    a = np.abs(x.astype(np.float64))
    i = np.searchsorted(g, a, side="right") - 1
    lo, hi = g[i], g[np.minimum(i + 1, g.size - 1)]
    oa = np.abs(out)
    assert np.all((oa == lo) | (oa == hi))
    assert np.all(np.sign(out)[oa > 0] == np.sign(x)[oa > 0])


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "e5m2"])
def test_probability_of_rounding_up_closed_form(orc, dtype):
    # over all 2^16 draws the count of "hi" is #{k : k < floor(f 2^16)} = floor(f 2^16):
    # the draw is added to the fraction's first 16 bits and the sum truncated
    g = _grid(dtype)
    rng = np.random.default_rng(5)
    ks = np.arange(65536, dtype=np.uint32)
    for _ in range(12):
        i = int(rng.integers(1, g.size - 2))
        lo, hi = g[i], g[i + 1]
        v = np.float32(lo + (hi - lo) * rng.random())
        if float(v) in (lo, hi):
            continue
        out = _code_value(orc.sr_with_draws(np.full(65536, v, np.float32), ks, dtype), dtype)
        n_hi = int((out == hi).sum())
        f = (Fraction(float(v)) - Fraction(lo)) / (Fraction(hi) - Fraction(lo))
        expect = (f * 65536).numerator // (f * 65536).denominator      # floor
        assert n_hi == expect
        # which draws round up: exactly the k below that count
        k_hi = np.nonzero(out == hi)[0]
        assert k_hi.tolist() == list(range(expect))
        if dtype == "bf16":
            assert Fraction(n_hi, 65536) == f   # exactly unbiased on bf16


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "e5m2"])
def test_unbiased_over_steps(orc, dtype):
    # mean of 10^4 SR draws (different steps) is within 4 sigma of v
    g = _grid(dtype)
    rng = np.random.default_rng(6)
    for _ in range(4):
        i = int(rng.integers(10, g.size - 10))
        lo, hi = g[i], g[i + 1]
        v = np.float32(lo + (hi - lo) * (0.1 + 0.8 * rng.random()))
        vals = np.array([_code_value(orc.sr_round(np.array([v]), dtype, seed=99, step=s, index_base=12345), dtype)[0]
                         for s in range(10000)])
        f = (float(v) - lo) / (hi - lo)
        sigma = (hi - lo) * np.sqrt(f * (1 - f) / vals.size)
        assert abs(vals.mean() - float(v)) < 4 * sigma


def test_special_values(orc):
    k = np.array([0, 65535], np.uint32)
    nan2 = np.array([np.nan, -np.nan], np.float32)
    assert orc.sr_with_draws(nan2, k, "bf16").tolist() == [0x7FC0, 0x7FC0]
    assert orc.sr_with_draws(nan2, k, "fp8").tolist() == [0x7F, 0x7F]
    big = np.array([448.0, 460.0, 1e9, np.inf, -448.0, -500.0, -np.inf], np.float32)
    assert orc.sr_with_draws(big, np.zeros(7, np.uint32), "fp8").tolist() == [126, 126, 126, 126, 254, 254, 254]
    m = np.float32(3.3895313892515355e38)     # largest finite bf16
    above = np.nextafter(m, np.float32(np.inf))
    out = orc.sr_with_draws(np.array([above, -above, np.inf, -np.inf], np.float32), np.zeros(4, np.uint32), "bf16")
    assert out.tolist() == [0x7F7F, 0xFF7F, 0x7F80, 0xFF80]
    # e4m3 subnormal range: 2^-10 sits halfway between 0 and 2^-9
    v = np.full(65536, 2.0 ** -10, np.float32)
    out = orc.sr_with_draws(v, np.arange(65536, dtype=np.uint32), "fp8")
    assert int((out == 1).sum()) == 32768 and int((out == 0).sum()) == 32768


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "e5m2"])
def test_sr_round_uses_element_draws(orc, dtype):
    rng = np.random.default_rng(8)
    x = (rng.standard_normal(1000) * 0.02).astype(np.float32)
    out = orc.sr_round(x, dtype, seed=5, step=9, index_base=777)
    k = orc.draw16(5, 9, 777, 1000)
    assert np.array_equal(out, orc.sr_with_draws(x, k, dtype))


def test_special_values_e5m2(orc):
    k = np.array([0, 65535], np.uint32)
    assert orc.sr_with_draws(np.array([np.nan, -np.nan], np.float32), k, "e5m2").tolist() == [0x7F, 0x7F]
    big = np.array([57344.0, 60000.0, 1e9, np.inf, -57344.0, -61000.0, -np.inf], np.float32)
    out = orc.sr_with_draws(big, np.zeros(7, np.uint32), "e5m2").tolist()
    assert out == [0x7B, 0x7B, 0x7B, 0x7C, 0xFB, 0xFB, 0xFC]        # finite saturates, inf stays inf
    # subnormal range: 2^-17 sits halfway between 0 and 2^-16
    v = np.full(65536, 2.0 ** -17, np.float32)
    out = orc.sr_with_draws(v, np.arange(65536, dtype=np.uint32), "e5m2")
    assert int((out == 1).sum()) == 32768 and int((out == 0).sum()) == 32768
