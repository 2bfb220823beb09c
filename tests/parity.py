"""Parity metrics between the CUDA path and the oracle (test helpers).

Tolerances (from the stated targets of the step):
  logits and dX: per-element relative error |a - b| / max(|b|, 0.01 rms(row of b))
                 at most 2e-2 (bf16 operands), 6e-2 (E4M3 operands) or 1.2e-1 (an
                 E5M2 gradient operand: one mantissa bit fewer, so the bound on a
                 term's rounding doubles).  Every comparison also records the max
                 and the 99.99th percentile under floors of 0.01 and 0.1 of the
                 row's rms (written to the file named by ELMO_PARITY_REPORT, one
                 JSON line per comparison, when that variable is set);
  gradient operands: each side's G is the correctly rounded operand of its own
                 logit (sigmoid correctly rounded to fp32, then G = s - y rounded
                 to nearest even onto bf16, or 2^8 G onto E4M3 / E5M2), checked
                 element by element; where the two logits (fp32 sums in
                 different orders) round to different operand codes, the oracle's
                 dX is corrected by exactly those terms before comparing, and
                 the label rows holding them are re-stepped from the GPU's
                 operands (the flip moves the whole row's update); operands
                 of the two sides never differ by more than one grid step;
  weights:       at least 99.9 % of elements within 1 grid ulp of the oracle
                 and |mean signed error| <= 0.05 ulp over every chunk;
  SR, Philox draws and top-k indices: bit-exact.
"""
import json
import os

import numpy as np

REL_TOL = {"bf16": 2e-2, "fp8": 6e-2, "fp8_ge5m2": 1.2e-1, "e5m2": 6e-2}


def weight_dtype(dtype):
    """The grid the weights of a head of `dtype` are stored on."""
    return {"bf16": "bf16", "fp8": "fp8", "fp8_ge5m2": "fp8", "e5m2": "e5m2"}[dtype]

FLOOR = 1e-2


def rel_err(a, b, axis=-1, floor=FLOOR):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    rms = np.sqrt(np.mean(b * b, axis=axis, keepdims=True))
    den = np.maximum(np.abs(b), floor * rms)
    den = np.where(den == 0, 1.0, den)
    return np.abs(a - b) / den


def error_report(a, b, axis=-1):
    """max and 99.99th percentile of the relative error under floors 0.01 and 0.1."""
    out = {}
    for f in (0.01, 0.1):
        e = rel_err(a, b, axis=axis, floor=f)
        out[f"floor{f}"] = {"max": float(e.max()) if e.size else 0.0,
                            "p99.99": float(np.quantile(e, 0.9999)) if e.size else 0.0}
    return out


def _record(entry):
    path = os.environ.get("ELMO_PARITY_REPORT")
    if not path:
        return
    test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    with open(path, "a") as f:
        f.write(json.dumps({"test": test, **entry}) + "\n")


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


def _worst_weights(gpu_codes, orc_codes, dtype, n=6):
    d = np.abs(ordinal(gpu_codes, dtype) - ordinal(orc_codes, dtype)).reshape(np.shape(gpu_codes)[0], -1)
    idx = np.argsort(d, axis=None)[::-1][:n]
    g = np.asarray(gpu_codes).reshape(d.shape)
    o = np.asarray(orc_codes).reshape(d.shape)
    return [(int(i // d.shape[1]), int(i % d.shape[1]), hex(int(g.flat[i])), hex(int(o.flat[i]))) for i in idx]


def assert_weights_close(gpu_codes, orc_codes, dtype, chunk_rows=None):
    within, worst = weight_parity(gpu_codes, orc_codes, dtype, chunk_rows)
    _record({"what": "weights", "within_1ulp": within, "mean_signed_err_ulp": worst})
    assert within >= 0.999, (f"only {within:.5%} of weights within 1 ulp; largest differences "
                             f"(row, col, gpu, oracle) {_worst_weights(gpu_codes, orc_codes, dtype)}")
    assert worst <= 0.05, (f"mean signed error {worst:.4f} ulp over a chunk; largest differences "
                           f"(row, col, gpu, oracle) {_worst_weights(gpu_codes, orc_codes, dtype)}")


def assert_rel_close(a, b, dtype, axis=-1, what="values"):
    rep = error_report(a, b, axis=axis)
    _record({"what": what, "dtype": dtype, **rep})
    e = rel_err(a, b, axis=axis)
    assert np.all(np.isfinite(e)), f"{what}: non-finite values"
    assert float(e.max()) <= REL_TOL[dtype], (f"{what}: max rel err {float(e.max()):.3e} > {REL_TOL[dtype]} "
                                              f"(report {rep})")


# ---------------------------------------------------------------- gradient operands
def operand_format(dtype):
    return {"bf16": "bf16", "fp8": "e4m3", "fp8_ge5m2": "e5m2", "e5m2": "e4m3"}[dtype]


def sigmoid_f32(z):
    """sigmoid(z) = 1 / (1 + e^-z) evaluated in double and rounded to fp32."""
    z64 = np.asarray(z, np.float32).astype(np.float64)
    with np.errstate(over="ignore"):
        return (1.0 / (1.0 + np.exp(-z64))).astype(np.float32)


def operand_of_logit(z, y, fmt):
    """The gradient operand value G that logit z and label y give: fp32
    g = sigmoid(z) - y, rounded to nearest even onto bf16, or 2^8 g onto the
    8-bit grid (the value returned has 2^-8 undone)."""
    import ml_dtypes
    g = (sigmoid_f32(z) - np.asarray(y, np.float32)).astype(np.float32)
    if fmt == "bf16":
        return g.astype(ml_dtypes.bfloat16).astype(np.float64)
    t = ml_dtypes.float8_e4m3fn if fmt == "e4m3" else ml_dtypes.float8_e5m2
    return (g * np.float32(256.0)).astype(np.float32).astype(t).astype(np.float64) / 256.0


def positives(rowptr, cols, L, B, l0=0, l1=None):
    """Y[l - l0, b] = 1 where label l is a positive of sample b."""
    l1 = L if l1 is None else l1
    Y = np.zeros((l1 - l0, B), np.float32)
    for b in range(B):
        c = np.asarray(cols[rowptr[b]:rowptr[b + 1]], np.int64)
        c = c[(c >= l0) & (c < l1)]
        Y[c - l0, b] = 1.0
    return Y


def weight_values(W, dtype):
    import ml_dtypes
    if dtype == "bf16":
        return np.asarray(W).view(ml_dtypes.bfloat16).astype(np.float64)
    if dtype == "e5m2":
        return np.asarray(W).view(ml_dtypes.float8_e5m2).astype(np.float64)
    return np.asarray(W).view(ml_dtypes.float8_e4m3fn).astype(np.float64)


def assert_operands_of_logits(G, Z, Y, dtype, what="G"):
    """Every operand G[l, b] is the correctly rounded operand of Z[l, b]."""
    want = operand_of_logit(Z, Y, operand_format(dtype))
    bad = ~((np.asarray(G, np.float64) == want) | (np.isnan(G) & np.isnan(want)))
    _record({"what": what + " self-consistency", "dtype": dtype, "elements": int(np.size(G)),
             "mismatches": int(bad.sum())})
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} operands are not the rounded operand "
                           f"of their logit (first at {np.argwhere(bad)[0].tolist()})")


def flip_corrected_dx(dx_orc, G_gpu, G_orc, W, w_dtype):
    """The oracle's dX with the terms of differing gradient operands replaced
    by the GPU's: dX[b, :] += (G_gpu - G_orc)[l, b] * w[l, :] for every (l, b)
    where the two differ (W: the old weight codes, decoded row by row).  G
    arrays are [labels, rows of dx_orc]."""
    dx = np.asarray(dx_orc, np.float64).copy()
    dG = np.asarray(G_gpu, np.float64) - np.asarray(G_orc, np.float64)
    ls, bs = np.nonzero(dG)
    for l, b in zip(ls, bs):
        dx[b] += dG[l, b] * weight_values(W[l], w_dtype)
    return dx, int(ls.size)


def operand_codes(G, dtype):
    """Grid codes (as ordinals) of gradient operand values G (2^-8 undone)."""
    import ml_dtypes
    fmt = operand_format(dtype)
    g = np.asarray(G, np.float32)
    if fmt == "bf16":
        return ordinal(g.astype(ml_dtypes.bfloat16).view(np.uint16), "bf16")
    t = ml_dtypes.float8_e4m3fn if fmt == "e4m3" else ml_dtypes.float8_e5m2
    return ordinal((g * np.float32(256.0)).astype(t).view(np.uint8), "fp8")


def x_operand(orc, X, dtype):
    """The X values the update's contraction uses: the bf16 inputs, or (8-bit
    heads) their E4M3 codes under the per-step scale s_X, divided by s_X."""
    Xf = orc.bf16_value(np.asarray(X, np.uint16))
    if dtype == "bf16":
        return Xf
    sx = np.float32(orc.fp8_x_scale(X))
    return orc.e4m3_value(orc.rne_e4m3((Xf * sx).astype(np.float32))) / sx


def flip_corrected_weights(orc, W, X, G_gpu, G_orc, W_new, lr, seed, step, dtype, l0=0):
    """The oracle's new weights with every label row whose gradient operands
    differ between the two sides re-stepped from the GPU's operands.  A
    differing operand is one grid step of G (a logit within rounding of a
    midpoint on one side); in an update W - lr G^T X that step moves the whole
    row by lr ulp(G) x, which can be many ulps of small weights.  The re-step
    follows the oracle's own arithmetic (fp32 products and sums in sample
    order, v = w - lr dw, the same 16-bit draws), checked first by
    re-stepping each such row from the oracle's operands and getting the
    oracle's codes back.  Rows of G and W_new are labels l0, l0 + 1, ...; W
    holds the old weights of the whole head.  Returns (weights, rows
    re-stepped)."""
    dG = np.asarray(G_gpu, np.float64) - np.asarray(G_orc, np.float64)
    rows = np.unique(np.nonzero(dG)[0])
    if rows.size == 0:
        return W_new, 0
    wd = weight_dtype(dtype)
    xv = x_operand(orc, X, dtype).astype(np.float32)
    d = xv.shape[1]
    out = np.array(W_new, copy=True)
    lr32 = np.float32(lr)

    def restep(l, g):
        dw = np.zeros(d, np.float32)
        for b in range(xv.shape[0]):
            dw = (dw + (np.float32(g[b]) * xv[b]).astype(np.float32)).astype(np.float32)
        v = (orc.w_value(W[l0 + l], wd).astype(np.float32) - (lr32 * dw).astype(np.float32)).astype(np.float32)
        return orc.sr_with_draws(v, orc.draw16(seed, step, int(l0 + l) * d, d), wd)

    for l in rows:
        assert np.array_equal(restep(l, G_orc[l]), W_new[l]), f"re-stepping label {l} does not reproduce the oracle"
        out[l] = restep(l, G_gpu[l])
    return out, int(rows.size)


def check_step(orc, W, X, rowptr, cols, lr, seed, step, dtype, Wg, dXg, Zg, Gg, chunk_rows=None,
               same_weights=True):
    """The GPU step (new weights Wg, dX dXg, logits Zg and operands Gg of the
    old weights) against the oracle's step on the same inputs.  same_weights
    False: the GPU stepped from its own earlier weights (a trajectory), which
    differ from W by stochastic-rounding decisions; the logits are then not
    compared (a weight one grid step apart moves a logit by x ulp(w), which a
    relative error against the row's rms floor does not absorb).  Returns the
    oracle's step (with W_ref, its weights with the flipped rows re-stepped:
    the start of the oracle's next step in a trajectory) and the flip count."""
    r = orc.train_step(W, X, rowptr, cols, lr, seed, step, dtype, want_zg=True)
    L, B = r["Z"].shape
    Y = positives(rowptr, cols, L, B)
    if same_weights:
        assert_rel_close(Zg, r["Z"], "bf16" if dtype == "bf16" else "fp8", axis=None, what="Z")
    assert_operands_of_logits(Gg, Zg, Y, dtype, what="G (GPU)")
    assert_operands_of_logits(r["G"], r["Z"], Y, dtype, what="G (oracle)")
    dx_ref, flips = flip_corrected_dx(r["dX"], Gg, r["G"], W, weight_dtype(dtype))
    steps = np.abs(operand_codes(Gg, dtype) - operand_codes(r["G"], dtype))
    w_ref, rows = flip_corrected_weights(orc, W, X, Gg, r["G"], r["W"], lr, seed, step, dtype)
    _record({"what": "G flips", "dtype": dtype, "elements": int(np.size(Gg)), "flips": flips,
             "largest_code_step": int(steps.max()) if steps.size else 0, "label_rows_restepped": rows})
    if same_weights:     # from different weights the logits, and so the operands, may differ more
        assert steps.size == 0 or int(steps.max()) <= 1, "the sides' gradient operands differ by more than one step"
    assert_rel_close(dXg, dx_ref, dtype, what="dX")
    assert_weights_close(Wg, w_ref, weight_dtype(dtype), chunk_rows=chunk_rows)
    r["W_ref"] = w_ref
    return r, flips
