"""Pins of the oracle's number grids and round-to-nearest conversions
against ml_dtypes / torch conversions (library routines)."""
import ml_dtypes
import numpy as np
import torch


def test_e4m3_decode_all_codes(orc):
    codes = np.arange(256, dtype=np.uint8)
    got = orc.e4m3_value(codes)
    ref = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float32)
    ref_t = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).float().numpy()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.array_equal(got[ok], ref_t[ok])
    assert np.nanmax(got) == 448.0 and np.nanmin(got[got > 0]) == 2.0 ** -9


def _rand_f32(rng, n, lo_exp, hi_exp):
    m = rng.random(n) + 1.0
    e = rng.integers(lo_exp, hi_exp, n)
    s = np.where(rng.random(n) < 0.5, -1.0, 1.0)
    return (s * np.ldexp(m, e)).astype(np.float32)


def test_rne_e4m3_matches_ml_dtypes(orc):
    rng = np.random.default_rng(0)
    grid = orc.e4m3_value(np.arange(127, dtype=np.uint8)).astype(np.float64)
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)          # exact ties
    x = np.concatenate([_rand_f32(rng, 20000, -14, 9), mids, -mids, grid.astype(np.float32),
                        np.array([0.0, -0.0, 447.9, 448.0, 2.0 ** -10, 2.0 ** -11], np.float32)])
    x = x[np.abs(x) <= 448]
    got = orc.rne_e4m3(x)
    ref = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(got, ref)
    # above the range the oracle saturates (satfinite)
    assert np.all(orc.rne_e4m3(np.array([449, 1e6, np.inf], np.float32)) == 126)
    assert np.all(orc.rne_e4m3(np.array([-449, -np.inf], np.float32)) == 0x80 | 126)


def test_rne_bf16_matches_torch(orc):
    rng = np.random.default_rng(1)
    x = np.concatenate([_rand_f32(rng, 50000, -140, 128),
                        rng.standard_normal(20000).astype(np.float32)])
    # exact ties: bf16 value + half ulp
    bits = rng.integers(0, 0x7F7F, 5000).astype(np.uint32) << 16
    ties = (bits | 0x8000).view(np.float32)
    x = np.concatenate([x, ties, -ties, np.array([0, -0.0, np.inf, -np.inf, 3.4e38], np.float32)])
    got = orc.rne_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


def test_fp8_x_scale_is_largest_fitting_power_of_two(orc):
    from synthetic import bf16_bits, bf16_value
    rng = np.random.default_rng(2)
    for scale in [1e-30, 1e-6, 0.03, 0.5, 1.0, 3.0, 448.0, 449.0, 1e5, 1e37]:
        X = bf16_bits(rng.standard_normal(64).astype(np.float32) * np.float32(scale))
        amax = float(np.abs(bf16_value(X)).max())
        s = orc.fp8_x_scale(X)
        e = np.log2(s)
        assert e == int(e)
        if -126 < e < 126:
            assert s * amax <= 448.0 < 2 * s * amax
    assert orc.fp8_x_scale(np.zeros(8, np.uint16)) == 1.0
    # a non-finite entry leaves X unscaled
    assert orc.fp8_x_scale(bf16_bits(np.array([1.0, np.inf], np.float32))) == 1.0


def test_e5m2_decode_all_codes(orc):
    codes = np.arange(256, dtype=np.uint8)
    got = orc.e5m2_value(codes)
    ref = codes.view(ml_dtypes.float8_e5m2).astype(np.float32)
    ref_t = torch.from_numpy(codes.copy()).view(torch.float8_e5m2).float().numpy()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.array_equal(got[ok], ref_t[ok])
    assert np.nanmax(got[np.isfinite(got)]) == 57344.0 and np.nanmin(got[got > 0]) == 2.0 ** -16
    assert got[0x7C] == np.inf and got[0xFC] == -np.inf


def test_rne_e5m2_matches_ml_dtypes(orc):
    rng = np.random.default_rng(1)
    grid = orc.e5m2_value(np.arange(0x7C, dtype=np.uint8)).astype(np.float64)   # finite magnitudes
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)                      # exact ties
    x = np.concatenate([_rand_f32(rng, 20000, -20, 16), mids, -mids, grid.astype(np.float32),
                        np.array([0.0, -0.0, 57343.0, 57344.0, 2.0 ** -17, 2.0 ** -18], np.float32)])
    x = x[np.abs(x) <= 57344]
    got = orc.rne_e5m2(x)
    ref = x.astype(ml_dtypes.float8_e5m2).view(np.uint8)
    assert np.array_equal(got, ref)
    # beyond the largest finite value the oracle saturates (satfinite); NaN -> 0x7F
    assert np.all(orc.rne_e5m2(np.array([61440, 1e9, np.inf], np.float32)) == 0x7B)
    assert np.all(orc.rne_e5m2(np.array([-61440, -np.inf], np.float32)) == 0xFB)
    assert orc.rne_e5m2(np.array([np.nan], np.float32))[0] == 0x7F
