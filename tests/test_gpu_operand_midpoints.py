"""Gradient operands at logits built to sit within a few fp32 ulps of the
points where the operand's rounding changes.

G = sigmoid(z) - y is rounded to nearest even onto the operand grid (bf16, or
2^8 G onto E4M3 / E5M2).  These tests build, for every (label, sample) pair,
a logit whose sigmoid lies next to a midpoint between two adjacent grid
values (for y = 0 and for y = 1), so that nearly every element falls inside
the kernels' uncertainty window and takes the exact per-element path.

Construction (exact in fp32): each sample owns P columns of X holding fixed
powers of two (bf16: three columns of 1; 8-bit heads: six columns of
decreasing scale), and each label's W entries in those columns are the parts
of the target logit, so that Z[l, b] = sum of exact products.  One more
column per sample holds X = 1 and W = 0: the step's update of that column is
W' = SR(0 - lr G[l, b]), and with lr chosen so that lr G lies on the weight
grid the stochastic rounding is exact, so W' exposes the operand the training
step itself formed (not only the inspection call's)."""
import numpy as np
import pytest
import torch

from tests.gpu_common import need_gpu, to_dev_i32, to_dev_u16, w_to_dev, w_to_host
from tests.parity import operand_format, operand_of_logit

pytestmark = pytest.mark.gpu


def _grid_values(fmt):
    import ml_dtypes
    if fmt == "bf16":
        c = np.arange(0, 0x7F80, dtype=np.uint16)
        return c.view(ml_dtypes.bfloat16).astype(np.float64)
    t = ml_dtypes.float8_e4m3fn if fmt == "e4m3" else ml_dtypes.float8_e5m2
    c = np.arange(0, 0x7F if fmt == "e4m3" else 0x7C, dtype=np.uint8)
    return c.view(t).astype(np.float64) / 256.0           # operand values (2^-8 undone)


def _midpoint_logits(fmt, y, zlo=-9.5, zhi=9.5, ulps=4):
    """fp32 logits within +-ulps of each logit whose sigmoid - y is a midpoint
    of the operand grid, for midpoints with logits in [zlo, zhi]."""
    g = _grid_values(fmt)
    if y:
        g = -g[::-1]                                       # G = s - 1 in (-1, 0]
    mid = 0.5 * (g[1:] + g[:-1])
    s = mid + y                                            # sigmoid at the midpoint
    ok = (s > 0) & (s < 1)
    z = np.log(s[ok] / (1.0 - s[ok]))
    z = z[(z >= zlo) & (z <= zhi)].astype(np.float32)
    out = [z]
    up, dn = z.copy(), z.copy()
    for _ in range(ulps):
        up = np.nextafter(up, np.float32(np.inf))
        dn = np.nextafter(dn, np.float32(-np.inf))
        out += [up.copy(), dn.copy()]
    return np.unique(np.concatenate(out))


def _parts(z, grid, scales):
    """Greedy split of each float64 value z into len(scales) terms
    part_j * scales[j] with part_j on `grid` (ml_dtypes type); returns the
    parts and whether the split is exact."""
    r = z.astype(np.float64).copy()
    parts = []
    for sc in scales:
        p = (r / sc).astype(grid)
        parts.append(p)
        r = r - p.astype(np.float64) * sc
    return parts, r == 0


def _layout(dtype):
    """(P, scales of X in the part columns, weight grid, lr, batch)"""
    import ml_dtypes
    if dtype == "bf16":
        return 3, [1.0, 1.0, 1.0], ml_dtypes.bfloat16, 1.0, 192
    # X = 1, 2^-4, 2^-8, 2^-12, 2^-15, 2^-17: the E4M3 operand 2^8 x stays exact (>= 2^-9)
    return 6, [1.0, 2.0**-4, 2.0**-8, 2.0**-12, 2.0**-15, 2.0**-17], ml_dtypes.float8_e4m3fn, 256.0, 96


@pytest.mark.parametrize("fused", ["1", "0"])
@pytest.mark.parametrize("dtype", ["bf16", "fp8", "fp8_ge5m2"])
def test_operands_next_to_rounding_midpoints(orc, dtype, fused, monkeypatch):
    """fused "0": the range-by-range kernels; "1": the persistent step."""
    need_gpu()
    monkeypatch.setenv("ELMO_STEP_FUSED", fused)
    import ml_dtypes
    import precision_label_chunk_b200 as elmo
    fmt = operand_format(dtype)
    P, scales, wgrid, lr, B = _layout(dtype)
    d, L = 768, 640                                        # five label tiles
    rng = np.random.default_rng(7)
    z0 = _midpoint_logits(fmt, 0)
    z1 = _midpoint_logits(fmt, 1)
    # positives: sample b has labels b % L and (3 b + 1) % L
    Y = np.zeros((L, B), np.float32)
    for b in range(B):
        Y[b % L, b] = 1.0
        Y[(3 * b + 1) % L, b] = 1.0
    target = np.where(Y > 0, rng.choice(z1, size=(L, B)), rng.choice(z0, size=(L, B))).astype(np.float32)
    parts, exact = _parts(target, wgrid, scales)
    X = np.zeros((B, d), np.float32)
    W = np.zeros((L, d), np.float64)
    for b in range(B):
        for j in range(P):
            X[b, b * P + j] = scales[j]
            W[:, b * P + j] = parts[j][:, b].astype(np.float64)
        X[b, P * B + b] = 1.0                              # the read-out column (W = 0 there)
    Xb = X.astype(ml_dtypes.bfloat16).view(np.uint16)
    Wc = W.astype(wgrid).view(np.uint16 if dtype == "bf16" else np.uint8)
    cols = np.concatenate([np.nonzero(Y[:, b])[0] for b in range(B)]).astype(np.int32)
    rowptr = np.concatenate([[0], np.cumsum((Y > 0).sum(axis=0))]).astype(np.int32)

    Wd = w_to_dev(Wc, dtype)
    h = elmo.elmo_init_head(Wd, dtype)
    Xd, rp, cl = to_dev_u16(Xb), to_dev_i32(rowptr), to_dev_i32(cols)
    Zd = torch.empty(L, B, device="cuda")
    Gd = torch.empty(L, B, device="cuda")
    elmo.elmo_forward_chunk(h, Xd, rp, cl, 0, L, Zd, Gd)
    dX = torch.empty(B, d, device="cuda")
    elmo.elmo_train_step_chunked(h, Xd, rp, cl, lr, 256, 5, 1, dX)
    elmo.elmo_sync_status(h)
    Z, G = Zd.cpu().numpy(), Gd.cpu().numpy()
    Wn = w_to_host(Wd, dtype)
    h.close()

    hit = Z == target
    assert hit.mean() > 0.9, f"only {hit.mean():.3f} of the built logits came out exactly"
    want = operand_of_logit(Z, Y, fmt)
    assert np.array_equal(G, want), f"inspection call: {int((G != want).sum())} operands differ"
    # the step's own operands, read back from the update of the read-out columns
    ro = Wn[:, P * B:P * B + B]
    if dtype == "bf16":
        Gstep = -((ro.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    else:
        Gstep = -ro.view(ml_dtypes.float8_e4m3fn).astype(np.float64) / lr
    bad = Gstep != want
    assert not bad.any(), (f"training step: {int(bad.sum())} of {bad.size} operands differ "
                           f"(first at {np.argwhere(bad)[0].tolist()})")
    # the construction does reach the rounding boundaries: the logits' fp32
    # neighbours round to different operands for a good share of elements
    up = operand_of_logit(np.nextafter(Z, np.float32(np.inf)), Y, fmt)
    dn = operand_of_logit(np.nextafter(Z, np.float32(-np.inf)), Y, fmt)
    assert np.mean((up != want) | (dn != want)) > 0.05
