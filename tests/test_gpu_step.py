"""The CUDA training step against the oracle (element-wise, seeded inputs)."""
import numpy as np
import pytest
import torch

from synthetic import make_labels, make_W_bf16, make_W_f32, make_X, workload
from tests.gpu_common import (need_gpu, run_step, run_step_with_operands, to_dev_i32, to_dev_u16, w_to_dev,
                               w_to_host)
from tests.parity import (assert_operands_of_logits, assert_rel_close, assert_weights_close, check_step, positives,
                          weight_parity)

pytestmark = pytest.mark.gpu


def _inputs(orc, w, step=0):
    X = make_X(w, step)
    rowptr, cols = make_labels(w, step)
    if w.dtype == "bf16":
        W = make_W_bf16(w)
    else:
        W = orc.sr_round(make_W_f32(w), "fp8", seed=0, step=2**64 - 1)
    return W, X, rowptr, cols


CASES = [
    ("tiny", {}),                                   # B=32, d=64, L=4096 (the tiny workload)
    ("tiny", {"dtype": "fp8"}),
    ("tiny", {"L": 1000, "d": 128, "B": 17}),       # ragged label tail, odd B
    ("tiny", {"L": 777, "d": 192, "B": 1, "dtype": "fp8"}),
    ("text500k_bf16", {"L": 3000, "B": 256}),       # full width and batch, several tiles
    ("product3m_fp8", {"L": 2500, "B": 256}),
]


@pytest.mark.parametrize("name,over", CASES)
def test_step_matches_oracle(orc, name, over):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload(name, **over)
    W, X, rowptr, cols = _inputs(orc, w)
    chunk = min(w.chunk, 1024)
    Wg, dXg, Zg, Gg = run_step_with_operands(elmo, W, X, rowptr, cols, w.lr, chunk, 0, 0, w.dtype)
    check_step(orc, W, X, rowptr, cols, w.lr, 0, 0, w.dtype, Wg, dXg, Zg, Gg, chunk_rows=chunk)


def _wide_logit_inputs(orc, dtype, L, B=256, d=768, seed=77):
    """X ~ N(0, 1) and W ~ N(0, 0.15^2): logits z ~ N(0, 4.2^2), so the gradient
    operand takes values over sigmoid's whole range, z < -5.5 (2^8 sigmoid < 1)
    and z > 5.5 (positives with 1 - sigmoid < 2^-8) included."""
    from synthetic import bf16_bits
    rng = np.random.default_rng(seed)
    X = bf16_bits(rng.standard_normal((B, d)).astype(np.float32))
    Wf = (0.15 * rng.standard_normal((L, d))).astype(np.float32)
    W = bf16_bits(Wf) if dtype == "bf16" else orc.sr_round(Wf, "fp8", seed=0, step=2**64 - 1)
    npos = 1 + rng.poisson(5, B)
    cols = np.concatenate([np.sort(rng.choice(L, k, replace=False)) for k in npos]).astype(np.int32)
    rowptr = np.concatenate([[0], np.cumsum(npos)]).astype(np.int32)
    return W, X, rowptr, cols


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "fp8_ge5m2"])
def test_step_wide_logits(orc, dtype):
    """B = 256, d = 768 over eight label tiles with logits spread over about
    +-15: G (through forward_chunk), dX and W against the oracle element by
    element, sigmoid's tails included."""
    need_gpu()
    import precision_label_chunk_b200 as elmo
    L = 1000
    W, X, rowptr, cols = _wide_logit_inputs(orc, dtype, L)
    Wg, dXg, Zg, Gg = run_step_with_operands(elmo, W, X, rowptr, cols, 0.05, 512, 3, 1, dtype)
    assert np.mean(Zg < -5.5) > 0.05 and np.mean(Zg > 5.5) > 0.05, "logits do not reach sigmoid's tails"
    check_step(orc, W, X, rowptr, cols, 0.05, 3, 1, dtype, Wg, dXg, Zg, Gg, chunk_rows=512)


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_forward_chunk_logits_and_gradients(orc, dtype):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("tiny", dtype=dtype, L=900, d=128, B=40)
    W, X, rowptr, cols = _inputs(orc, w)
    l0, l1 = 100, 900
    Wd = w_to_dev(W, dtype)
    h = elmo.elmo_init_head(Wd, dtype)
    Z = torch.empty(l1 - l0, w.B, device="cuda")
    G = torch.empty(l1 - l0, w.B, device="cuda")
    elmo.elmo_forward_chunk(h, to_dev_u16(X), to_dev_i32(rowptr), to_dev_i32(cols), l0, l1, Z, G)
    elmo.elmo_sync_status(h)
    r = orc.train_step(W, X, rowptr, cols, 0.0, 0, 0, dtype, l0=l0, l1=l1, want_zg=True)
    assert_rel_close(Z.cpu().numpy(), r["Z"], dtype, axis=None, what="Z")
    # G is the correctly rounded operand of each side's own logit; where the
    # logits agree the operands are equal
    Y = positives(rowptr, cols, w.L, w.B, l0, l1)
    g, go, z = G.cpu().numpy(), r["G"], Z.cpu().numpy()
    assert_operands_of_logits(g, z, Y, dtype)
    same = z == r["Z"]
    assert np.array_equal(g[same], go[same])
    # W untouched
    assert np.array_equal(w_to_host(Wd, dtype), W)
    h.close()


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_weights_independent_of_chunk(orc, dtype):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("tiny", dtype=dtype, L=1500, d=128, B=24)
    W, X, rowptr, cols = _inputs(orc, w)
    outs = [run_step(elmo, W, X, rowptr, cols, w.lr, c, 4, 9, dtype) for c in (1500, 512, 129, 64)]
    for Wg, dXg in outs[1:]:
        assert np.array_equal(Wg, outs[0][0])
        assert np.allclose(dXg, outs[0][1], rtol=1e-4, atol=1e-5)


def test_empty_labels_and_zero_lr(orc):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("tiny", L=600, d=64, B=8)
    W, X, _, _ = _inputs(orc, w)
    rowptr = np.zeros(w.B + 1, np.int32)
    cols = np.zeros(0, np.int32)
    Wg, dXg, Zg, Gg = run_step_with_operands(elmo, W, X, rowptr, cols, 0.0, 256, 1, 1, "bf16")
    vals = lambda a: (a.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(vals(Wg), vals(W))
    check_step(orc, W, X, rowptr, cols, 0.0, 1, 1, "bf16", Wg, dXg, Zg, Gg)


def test_malformed_labels_report_edata():
    need_gpu()
    import precision_label_chunk_b200 as elmo
    W = torch.zeros(256, 64, dtype=torch.bfloat16, device="cuda")
    h = elmo.elmo_init_head(W, "bf16")
    X = torch.zeros(2, 64, dtype=torch.bfloat16, device="cuda")
    dX = torch.empty(2, 64, device="cuda")
    rowptr = torch.tensor([0, 1, 2], dtype=torch.int32, device="cuda")
    cols = torch.tensor([3, 256], dtype=torch.int32, device="cuda")      # 256 is out of range
    elmo.elmo_train_step_chunked(h, X, rowptr, cols, 0.1, 128, 0, 0, dX)
    with pytest.raises(elmo.ElmoError) as ei:
        elmo.elmo_sync_status(h)
    assert ei.value.status == 6
    elmo.elmo_sync_status(h)                      # cleared
    bad_ptr = torch.tensor([0, 2, 1], dtype=torch.int32, device="cuda")
    elmo.elmo_train_step_chunked(h, X, bad_ptr, cols, 0.1, 128, 0, 0, dX)
    with pytest.raises(elmo.ElmoError):
        elmo.elmo_sync_status(h)
    with pytest.raises(elmo.ElmoError):       # B above the limit
        elmo.elmo_train_step_chunked(h, torch.zeros(300, 64, dtype=torch.bfloat16, device="cuda"),
                                     torch.zeros(301, dtype=torch.int32, device="cuda"), cols, 0.1, 128, 0, 0,
                                     torch.empty(300, 64, device="cuda"))
    h.close()


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_multistep_trajectory(orc, dtype):
    # GPU and oracle each run their own 4-step trajectory from the same start;
    # SR decisions that differ by summation order stay rare and unbiased.  A
    # gradient operand whose logit lies within rounding of a midpoint may take
    # either neighbour; the oracle's next step starts from its weights with
    # those label rows re-stepped from the GPU's (checked) operands, so that a
    # boundary choice made at one step is not counted again at the next
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("tiny", dtype=dtype, L=1200, d=128, B=32)
    W, _, _, _ = _inputs(orc, w)
    Wd = w_to_dev(W, dtype)
    h = elmo.elmo_init_head(Wd, dtype)
    dX = torch.empty(w.B, w.d, device="cuda")
    Z = torch.empty(w.L, w.B, device="cuda")
    G = torch.empty(w.L, w.B, device="cuda")
    Wo = W.copy()
    for s in range(4):
        X = make_X(w, s)
        rowptr, cols = make_labels(w, s)
        Xd, rp, cl = to_dev_u16(X), to_dev_i32(rowptr), to_dev_i32(cols)
        elmo.elmo_forward_chunk(h, Xd, rp, cl, 0, w.L, Z, G)
        elmo.elmo_train_step_chunked(h, Xd, rp, cl, w.lr, 512, 0, s, dX)
        elmo.elmo_sync_status(h)
        r, _ = check_step(orc, Wo, X, rowptr, cols, w.lr, 0, s, dtype, w_to_host(Wd, dtype), dX.cpu().numpy(),
                          Z.cpu().numpy(), G.cpu().numpy(), chunk_rows=512, same_weights=(s == 0))
        Wo = r["W_ref"]       # the oracle continues with the rounding-boundary choices the GPU made
    h.close()


def test_resume_is_exact(orc):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("tiny", dtype="fp8", L=700, d=128, B=16)
    W, _, _, _ = _inputs(orc, w)

    def run(Wstart, steps):
        Wd = w_to_dev(Wstart, "fp8")
        h = elmo.elmo_init_head(Wd, "fp8")
        dX = torch.empty(w.B, w.d, device="cuda")
        for s in steps:
            rp, cl = make_labels(w, s)
            elmo.elmo_train_step_chunked(h, to_dev_u16(make_X(w, s)), to_dev_i32(rp), to_dev_i32(cl), w.lr, 256, 3,
                                         s, dX)
        elmo.elmo_sync_status(h)
        out = w_to_host(Wd, "fp8").copy()
        h.close()
        return out

    straight = run(W, range(6))
    half = run(W, range(3))
    assert np.array_equal(run(half, range(3, 6)), straight)


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_step_special_weights(orc, dtype):
    """Infinities, NaNs, the largest finite values, subnormals and -0 among the
    weights take the update's exact per-element path: those weights get the
    oracle's codes exactly (a NaN weight makes its label's logits and gradient
    NaN, so its whole row becomes NaN on both sides); the other rows keep the
    usual statistical agreement."""
    need_gpu()
    import ml_dtypes
    import precision_label_chunk_b200 as elmo
    w = workload("tiny", dtype=dtype, L=600, d=128, B=24)
    W, X, rowptr, cols = _inputs(orc, w)
    specials = {"bf16": [0x7F80, 0xFF80, 0x7FC0, 0x7F7F, 0xFF7F, 0x7F00, 0x0001, 0x8000],
                "fp8": [0x7F, 0xFF, 0x7E, 0xFE, 0x01, 0x80, 0x7D, 0x08]}[dtype]
    pos = [(3 + 70 * i, (13 * i) % w.d) for i in range(len(specials))]
    W = W.copy()
    for (l, j), c in zip(pos, specials):
        W[l, j] = c
    Wg, _ = run_step(elmo, W, X, rowptr, cols, w.lr, 256, 7, 3, dtype)
    r = orc.train_step(W, X, rowptr, cols, w.lr, 7, 3, dtype)
    for (l, j), c in zip(pos, specials):
        assert Wg[l, j] == r["W"][l, j], f"special weight {c:#x} at ({l}, {j}): {Wg[l, j]:#x} vs {r['W'][l, j]:#x}"
    as_f = (lambda a: a.view(ml_dtypes.bfloat16).astype(np.float32)) if dtype == "bf16" else \
           (lambda a: a.view(ml_dtypes.float8_e4m3fn).astype(np.float32))
    nan_g, nan_o = np.isnan(as_f(Wg)), np.isnan(as_f(r["W"]))
    assert np.array_equal(nan_g, nan_o)
    finite_rows = ~np.any(~np.isfinite(as_f(r["W"])), axis=1)
    assert_weights_close(Wg[finite_rows], r["W"][finite_rows], dtype)


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_step_widest_embedding(orc, dtype):
    """d = 4096, the largest supported width: kernel A then streams X and W
    k-blocks (neither fits shared memory or TMEM as a resident operand), and
    kernel B runs 32 d-slices per label tile."""
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("tiny", dtype=dtype, L=520, d=4096, B=12)
    W, X, rowptr, cols = _inputs(orc, w)
    Wg, dXg, Zg, Gg = run_step_with_operands(elmo, W, X, rowptr, cols, w.lr, 256, 2, 5, dtype)
    check_step(orc, W, X, rowptr, cols, w.lr, 2, 5, dtype, Wg, dXg, Zg, Gg, chunk_rows=256)


def test_step_most_positives(orc):
    """nnz = 32768, the largest label list a step takes (256 samples x 128
    positives, every label tile crowded), on a small head."""
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("tiny", dtype="fp8", L=4096, d=128, B=256)
    W, X, _, _ = _inputs(orc, w)
    rng = np.random.default_rng(11)
    cols = np.concatenate([np.sort(rng.choice(w.L, 128, replace=False)) for _ in range(w.B)]).astype(np.int32)
    rowptr = (np.arange(w.B + 1) * 128).astype(np.int32)
    assert cols.size == 32768
    Wg, dXg, Zg, Gg = run_step_with_operands(elmo, W, X, rowptr, cols, w.lr, 1024, 3, 3, "fp8")
    check_step(orc, W, X, rowptr, cols, w.lr, 3, 3, "fp8", Wg, dXg, Zg, Gg, chunk_rows=1024)


def test_step_largest_label_index(orc):
    """L = 2^24 - 1, the most labels a head takes (the positive key packs the
    label in 24 bits): weights of the last labels, where the key's top bits
    are set, against the oracle on that range."""
    need_gpu()
    import precision_label_chunk_b200 as elmo
    from synthetic import bf16_bits
    L, d, B = 2**24 - 1, 64, 4
    rng = np.random.default_rng(5)
    X = bf16_bits(rng.standard_normal((B, d)).astype(np.float32))
    cols = np.array([L - 1, L - 200, 0, L - 1, L - 150, 7, L - 3], np.int32)
    rowptr = np.array([0, 2, 3, 5, 7], np.int32)
    Wd = torch.empty(L, d, dtype=torch.int16, device="cuda")
    h = elmo.elmo_init_head(Wd, "bf16", fill=True, init_std=0.02, seed=1)
    W0 = w_to_host(Wd, "bf16").copy()
    dX = torch.empty(B, d, device="cuda")
    elmo.elmo_train_step_chunked(h, to_dev_u16(X), to_dev_i32(rowptr), to_dev_i32(cols), 0.5, 1 << 20, 0, 9, dX)
    elmo.elmo_sync_status(h)
    l0 = L - 256
    r = orc.train_step(W0, X, rowptr, cols, 0.5, 0, 9, "bf16", l0=l0, l1=L, want_dx=False, L=L)
    assert_weights_close(w_to_host(Wd[l0:], "bf16"), r["W"], "bf16")
    h.close()
