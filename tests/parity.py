"""Parity metrics between the CUDA path and the oracle (test helpers).

Tolerances (from the stated targets of the step):
  logits and dX: per-element relative error |a - b| / max(|b|, 0.1 rms(row of b))
                 at most 2e-2 (bf16 operands), 6e-2 (E4M3 operands) or 1.2e-1 (an
                 E5M2 gradient operand: one more bit of spacing, so one flipped
                 operand moves a term twice as far).  The floor
                 of a tenth of the row's rms absorbs a gradient operand that the two
                 sides legitimately round to different grid neighbours (their fp32
                 logits or sigmoids differ in the last bit at a rounding midpoint):
                 that moves one term of dX by ulp(G) |w| (2^-8 |w| for bf16, 2^-4 |w|
                 for E4M3), which a tolerance relative to a near-zero element could
                 not absorb;
  weights:       at least 99.9 % of elements within 1 grid ulp of the oracle
                 and |mean signed error| <= 0.05 ulp over every chunk;
  SR, Philox draws and top-k indices: bit-exact.
"""
import numpy as np

REL_TOL = {"bf16": 2e-2, "fp8": 6e-2, "fp8_ge5m2": 1.2e-1}


FLOOR = 0.1


def rel_err(a, b, axis=-1):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    rms = np.sqrt(np.mean(b * b, axis=axis, keepdims=True))
    den = np.maximum(np.abs(b), FLOOR * rms)
    den = np.where(den == 0, 1.0, den)
    return np.abs(a - b) / den


def ordinal(codes, dtype):
    """Grid codes -> integers that step by one per grid point (+-0 -> 0)."""
    c = np.asarray(codes).astype(np.int64)
    if dtype == "bf16":
        mag, neg = c & 0x7FFF, (c & 0x8000) != 0
    else:
        mag, neg = c & 0x7F, (c & 0x80) != 0
    return np.where(neg, -mag, mag)


def weight_parity(gpu_codes, orc_codes, dtype, chunk_rows=None):
    """(fraction within 1 ulp, max |mean signed error| over chunks of rows)."""
    d = ordinal(gpu_codes, dtype) - ordinal(orc_codes, dtype)
    within = float(np.mean(np.abs(d) <= 1))
    d2 = d.reshape(d.shape[0], -1)
    rows = d2.shape[0]
    step = rows if chunk_rows is None else max(1, chunk_rows)
    worst = 0.0
    for a in range(0, rows, step):
        worst = max(worst, abs(float(np.mean(d2[a:a + step]))))
    return within, worst


def assert_weights_close(gpu_codes, orc_codes, dtype, chunk_rows=None):
    within, worst = weight_parity(gpu_codes, orc_codes, dtype, chunk_rows)
    assert within >= 0.999, f"only {within:.5%} of weights within 1 ulp"
    assert worst <= 0.05, f"mean signed error {worst:.4f} ulp over a chunk"


def assert_rel_close(a, b, dtype, axis=-1, what="values"):
    e = rel_err(a, b, axis=axis)
    assert np.all(np.isfinite(e)), f"{what}: non-finite values"
    assert float(e.max()) <= REL_TOL[dtype], f"{what}: max rel err {float(e.max()):.3e} > {REL_TOL[dtype]}"
