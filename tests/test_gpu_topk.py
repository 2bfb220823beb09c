"""The CUDA top-k against the oracle: indices bit-exact, ties to the lower index."""
import ml_dtypes
import numpy as np
import pytest
import torch

from synthetic import bf16_bits, make_W_f32, make_X, workload
from tests.gpu_common import need_gpu, to_dev_u16, w_to_dev

pytestmark = pytest.mark.gpu


def _gpu_topk(elmo, W, X, k, chunk, dtype):
    Wd = w_to_dev(W, dtype)
    h = elmo.elmo_init_head(Wd, dtype)
    idx = torch.empty(X.shape[0], k, dtype=torch.int32, device="cuda")
    sc = torch.empty(X.shape[0], k, dtype=torch.float32, device="cuda")
    elmo.elmo_topk_predict(h, to_dev_u16(X), k, chunk, idx, sc)
    torch.cuda.synchronize()
    out = idx.cpu().numpy(), sc.cpu().numpy()
    h.close()
    return out


@pytest.mark.parametrize("dtype,L,d,B,k", [("fp8", 5000, 128, 64, 5), ("bf16", 3000, 64, 33, 7),
                                           ("fp8", 20000, 768, 16, 5), ("fp8", 700, 256, 5, 64)])
def test_topk_matches_oracle(orc, dtype, L, d, B, k):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("topk5_3m_fp8", L=L, d=d, B=B)
    X = make_X(w, 0)
    wf = make_W_f32(w)
    W = orc.sr_round(wf, dtype, 0, 2**64 - 1)
    for chunk in (L, 1024):
        idx, sc = _gpu_topk(elmo, W, X, k, chunk, dtype)
        ri, rs = orc.topk(W, X, k, dtype)
        assert np.array_equal(idx, ri)
        assert np.array_equal(sc.view(np.uint32), rs.view(np.uint32))


def test_topk_exact_ties(orc):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    rng = np.random.default_rng(5)
    L, d, B, k = 4096, 128, 24, 8
    xv = (rng.integers(-4, 5, (B, d)) / 4).astype(np.float32)
    wv = (rng.integers(-4, 5, (L, d)) / 32).astype(np.float32)
    for a, b in [(10, 3000), (10, 4095), (700, 701), (5, 4000)]:
        wv[b] = wv[a]
    # make the duplicated rows the best for every sample
    wv[[10, 3000, 4095, 700, 701, 5, 4000]] = np.sign(xv[0]) * 0.125
    X = bf16_bits(xv)
    W = wv.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    idx, sc = _gpu_topk(elmo, W, X, k, 1000, "fp8")
    ri, rs = orc.topk(W, X, k, "fp8")
    assert np.array_equal(idx, ri)
    assert np.array_equal(sc, rs)


def _topk_dev(elmo, Wd, h, X, k, chunk=131072):
    idx = torch.empty(X.shape[0], k, dtype=torch.int32, device="cuda")
    sc = torch.empty(X.shape[0], k, dtype=torch.float32, device="cuda")
    elmo.elmo_topk_predict(h, to_dev_u16(X), k, chunk, idx, sc)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), sc.cpu().numpy()


@pytest.mark.parametrize("dtype,L,d,B,k", [("bf16", 6000, 768, 40, 5), ("fp8", 9001, 768, 300, 17),
                                           ("fp8", 65, 64, 3, 5), ("bf16", 130, 192, 129, 64),
                                           ("fp8", 40000, 512, 1024, 1)])
def test_topk_tensor_core_screening_matches_oracle(orc, dtype, L, d, B, k, monkeypatch):
    """Shapes that stress the screening layout: the widest A operand (d = 768),
    several query panels with a partial last one, heads smaller than a
    candidate list, k above 16 (64 candidates per range) and k = 1.  The
    result must equal the oracle's, and the CUDA-core path's."""
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("topk5_3m_fp8", L=L, d=d, B=B)
    X = make_X(w, 3)
    W = orc.sr_round(make_W_f32(w), dtype, 1, 2**64 - 1)
    Wd = w_to_dev(W, dtype)
    h = elmo.elmo_init_head(Wd, dtype)
    idx, sc = _topk_dev(elmo, Wd, h, X, k)
    rows = np.arange(B) if B <= 64 else np.array([0, 1, 127, 128, B // 2, B - 1])
    ri, rs = orc.topk(W, X, k, dtype, rows=rows)
    assert np.array_equal(idx[rows], ri)
    assert np.array_equal(sc[rows].view(np.uint32), rs.view(np.uint32))
    monkeypatch.setenv("ELMO_TOPK_SIMT", "1")
    si, ss = _topk_dev(elmo, Wd, h, X, k)
    assert np.array_equal(si, idx)
    assert np.array_equal(ss.view(np.uint32), sc.view(np.uint32))
    h.close()


@pytest.mark.parametrize("case", ["nan_weight", "inf_query"])
def test_topk_uncertified_rows_take_exact_path(orc, case):
    """A NaN weight leaves no finite bound on |W|: every row must be recomputed
    exactly (NaN scores rank last).  An infinite query value voids that row's
    bound only."""
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("topk5_3m_fp8", L=3000, d=128, B=20)
    X = make_X(w, 4)
    W = orc.sr_round(make_W_f32(w), "fp8", 2, 2**64 - 1)
    if case == "nan_weight":
        W[17, 5] = 0x7F
    else:
        X[3, 9] = 0x7F80
    Wd = w_to_dev(W, "fp8")
    h = elmo.elmo_init_head(Wd, "fp8")
    idx, sc = _topk_dev(elmo, Wd, h, X, 5)
    ri, rs = orc.topk(W, X, 5, "fp8")
    assert np.array_equal(idx, ri)
    assert np.array_equal(sc.view(np.uint32), rs.view(np.uint32))
    h.close()


@pytest.mark.parametrize("B,k,L", [(1024, 5, 3_000_000), (7, 64, 100), (1, 1, 10)])
def test_precision_at_k_matches_oracle(orc, B, k, L):
    """P@1..P@k on the GPU equals the oracle's value rounded to fp32, on seeded
    predictions (distinct labels per row) and the workload's label law."""
    need_gpu()
    import precision_label_chunk_b200 as elmo
    from synthetic import make_labels
    rng = np.random.default_rng(B * 131 + k)
    w = workload("product3m_fp8", L=L, B=B)
    rowptr, cols = make_labels(w, 1)
    # predictions: mostly positives of the row at random ranks, the rest random labels
    idx = np.zeros((B, k), np.int32)
    for b in range(B):
        pos = cols[rowptr[b]:rowptr[b + 1]]
        cand = np.concatenate([rng.permutation(pos)[: rng.integers(0, min(k, pos.size) + 1)],
                               rng.choice(L, size=min(2 * k, L), replace=False)])
        _, first = np.unique(cand, return_index=True)
        row = cand[np.sort(first)][:k]
        idx[b, : row.size] = rng.permutation(row)
        if row.size < k:
            idx[b, row.size:] = -1
    p = torch.empty(k, dtype=torch.float32, device="cuda")
    elmo.elmo_precision_at_k(torch.from_numpy(idx).cuda(), torch.from_numpy(rowptr).cuda(),
                             torch.from_numpy(cols).cuda(), p)
    want = orc.precision_at_k(idx, rowptr, cols).astype(np.float32)
    assert np.array_equal(p.cpu().numpy(), want)


@pytest.mark.parametrize("dtype,L", [("fp8", 3_000_000), ("bf16", 500_000)])
def test_screening_error_within_a_quarter_of_the_bound(orc, dtype, L):
    """The certificate assumes every accumulating MMA is off by at most 2^-20 of
    the sum of its products' magnitudes.  Measured on a full 131,072-label
    range of a workload-sized head: the screening scores stay within a quarter
    of each row's bound of the exact chain scores, and within a quarter of the
    per-element form of the same model (each label's own sum of |x w|)."""
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("topk5_3m_fp8", L=L, dtype=dtype)
    Wd = torch.empty(w.L, w.d, dtype=torch.uint8 if dtype == "fp8" else torch.int16, device="cuda")
    h = elmo.elmo_init_head(Wd, dtype, fill=True, init_std=0.02, seed=0)
    X = make_X(w, 0)
    l0 = (w.L // 2) // 128 * 128
    l1 = l0 + 131072
    rows = [0, 1, 255, 511, 1023]
    Xs = X[rows]
    S = torch.empty(len(rows), l1 - l0, device="cuda")
    bound = torch.empty(len(rows), device="cuda")
    elmo.elmo_topk_screen_scores(h, to_dev_u16(Xs), l0, l1, S, bound)
    torch.cuda.synchronize()
    Wh = Wd.cpu().numpy().view(np.uint8 if dtype == "fp8" else np.uint16)
    exact = orc.scores(Wh, Xs, np.arange(len(rows)), l0, l1, dtype)
    err = np.abs(S.cpu().numpy().astype(np.float64) - exact.astype(np.float64))
    bnd = bound.cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(bnd)) and np.all(bnd > 0)
    worst = (err.max(axis=1) / bnd)
    assert worst.max() <= 0.25, f"screening error reaches {worst.max():.3f} of the certificate's bound"
    # per element: nsteps 2^-20 sum|q w| (+ the E4M3 split's residual, + the chain's own error)
    xv = (Xs.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    wv = (Wh[l0:l1].view(ml_dtypes.float8_e4m3fn) if dtype == "fp8" else Wh[l0:l1].view(ml_dtypes.bfloat16))
    absw = np.abs(wv.astype(np.float32))
    mag = (np.abs(xv).astype(np.float32) @ absw.T).astype(np.float64) * (1 + 2.0 ** -16)   # sum_j |x_j w_lj|
    nsteps = (2 if dtype == "fp8" else 1) * (w.d * (1 if dtype == "fp8" else 2) // 128) * 4
    model = (nsteps * 2.0 ** -20 + 1.01 * w.d * 2.0 ** -24) * mag
    if dtype == "fp8":
        # the lo part of the E4M3 split is exact unless below 2^-9 (in scaled units):
        # residual at most 2^-10 / s_b per element
        s_b = np.array([2.0 ** np.floor(np.log2(448.0 / np.abs(x).max())) for x in xv])
        model += (2.0 ** -10 / s_b)[:, None] * absw.sum(axis=1)[None, :]
    ratio = err / np.maximum(model, 1e-30)
    assert ratio.max() <= 0.25, f"screening error reaches {ratio.max():.3f} of the per-element model"
    h.close()
