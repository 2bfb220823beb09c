"""A head with E5M2 weights (ELMO_FP8_E5M2): X and the gradient operand in
E4M3, the weights stored and stochastically rounded on the E5M2 grid.  The
step (each kernel-A variant, the persistent step), top-k and the no-alloc
entry against the oracle's E5M2 head."""
import os

import numpy as np
import pytest
import torch

from synthetic import make_labels, make_W_f32, make_X, workload
from tests.gpu_common import need_gpu, run_step_with_operands, to_dev_i32, to_dev_u16, w_to_dev, w_to_host
from tests.parity import assert_rel_close, assert_weights_close, check_step

pytestmark = pytest.mark.gpu
DT = "e5m2"


def _inputs(orc, w, step=0):
    X = make_X(w, step)
    rowptr, cols = make_labels(w, step)
    W = orc.sr_round(make_W_f32(w), "e5m2", seed=0, step=2**64 - 1)      # E5M2 codes
    return W, X, rowptr, cols


CASES = [
    ("tiny", {"L": 1000, "d": 128, "B": 17}),             # persistent step, one M-block, ragged tail
    ("product3m_fp8", {"L": 2500, "B": 256}),             # persistent step, two M-blocks (the workload's shape)
    ("product3m_fp8", {"L": 900, "d": 1024, "B": 256}),   # resident-X panel (d > 768)
    ("tiny", {"L": 600, "d": 4096, "B": 64}),             # streaming kernel A (no panel fits)
]


@pytest.mark.parametrize("name,over", CASES)
def test_e5m2_head_step_matches_oracle(orc, name, over):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload(name, dtype="fp8", **over)
    W, X, rowptr, cols = _inputs(orc, w)
    Wg, dXg, Zg, Gg = run_step_with_operands(elmo, W, X, rowptr, cols, w.lr, 512, 0, 0, DT)
    r, _ = check_step(orc, W, X, rowptr, cols, w.lr, 0, 0, DT, Wg, dXg, Zg, Gg, chunk_rows=512)
    # and the weights are on the E5M2 grid, not E4M3's
    r4 = orc.train_step(orc.sr_round(make_W_f32(w), "fp8", 0, 2**64 - 1), X, rowptr, cols, w.lr, 0, 0, "fp8")
    assert not np.array_equal(r["W"], r4["W"])


def test_e5m2_head_fill_matches_oracle_rounding(orc):
    """The device fill draws its normal values with the device's transcendental
    functions; its rounding onto E5M2 is checked on values the test recovers:
    every stored code is a finite E5M2 value near N(0, 0.02^2)."""
    need_gpu()
    import ml_dtypes
    import precision_label_chunk_b200 as elmo
    Wd = torch.empty(4096, 256, dtype=torch.uint8, device="cuda")
    h = elmo.elmo_init_head(Wd, DT, fill=True, init_std=0.02, seed=3)
    torch.cuda.synchronize()
    v = Wd.cpu().numpy().view(ml_dtypes.float8_e5m2).astype(np.float64)
    assert np.all(np.isfinite(v))
    assert abs(v.std() - 0.02) < 0.002 and abs(v.mean()) < 0.001
    h.close()


def test_e5m2_head_weights_identical_on_both_step_paths(orc):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("product3m_fp8", L=1500, B=256)
    W, _, _, _ = _inputs(orc, w)
    outs = []
    for fused in ("0", "1"):
        os.environ["ELMO_STEP_FUSED"] = fused
        try:
            Wd = w_to_dev(W, "fp8")
            h = elmo.elmo_init_head(Wd, DT)
            dX = torch.empty(w.B, w.d, device="cuda")
            for s in range(3):
                rp, cl = make_labels(w, s)
                elmo.elmo_train_step_chunked(h, to_dev_u16(make_X(w, s)), to_dev_i32(rp), to_dev_i32(cl), w.lr, 512,
                                             0, s, dX)
            elmo.elmo_sync_status(h)
            outs.append(w_to_host(Wd, "fp8").copy())
            h.close()
        finally:
            os.environ.pop("ELMO_STEP_FUSED", None)
    assert np.array_equal(outs[0], outs[1])


@pytest.mark.parametrize("L,d,B,k", [(5000, 128, 64, 5), (20000, 768, 16, 5)])
def test_e5m2_head_topk_matches_oracle(orc, L, d, B, k):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("topk5_3m_fp8", L=L, d=d, B=B)
    X = make_X(w, 0)
    W = orc.sr_round(make_W_f32(w), "e5m2", 0, 2**64 - 1)
    Wd = w_to_dev(W, "fp8")
    h = elmo.elmo_init_head(Wd, DT)
    idx = torch.empty(B, k, dtype=torch.int32, device="cuda")
    sc = torch.empty(B, k, dtype=torch.float32, device="cuda")
    elmo.elmo_topk_predict(h, to_dev_u16(X), k, 4096, idx, sc)
    torch.cuda.synchronize()
    ri, rs = orc.topk(W, X, k, DT)
    assert np.array_equal(idx.cpu().numpy(), ri)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    h.close()


def test_e5m2_head_noalloc_matches_head_step(orc):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("product3m_fp8", L=3000, B=256)
    W, X, rowptr, cols = _inputs(orc, w)
    Wa, Wb = w_to_dev(W, "fp8"), w_to_dev(W, "fp8")
    Xd, rp, cl = to_dev_u16(X), to_dev_i32(rowptr), to_dev_i32(cols)
    dXa = torch.empty(w.B, w.d, device="cuda")
    dXb = torch.empty(w.B, w.d, device="cuda")
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    h = elmo.elmo_init_head(Wa, DT)
    elmo.elmo_train_step_chunked(h, Xd, rp, cl, w.lr, 1024, 0, 0, dXa)
    elmo.elmo_sync_status(h)
    h.close()
    elmo.elmo_train_step_noalloc(Wb, DT, Xd, rp, cl, w.lr, 1024, 0, 0, dXb, status)
    torch.cuda.synchronize()
    assert int(status[0]) == 0
    assert torch.equal(Wa, Wb)
    r = orc.train_step(W, X, rowptr, cols, w.lr, 0, 0, DT)
    assert_weights_close(w_to_host(Wb, "fp8"), r["W"], "e5m2", chunk_rows=1024)
    assert_rel_close(dXb.cpu().numpy(), r["dX"], DT, what="dX")
