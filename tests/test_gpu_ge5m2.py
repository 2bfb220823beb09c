"""The E4M3 step with an E5M2 gradient operand (ELMO_FP8_E4M3_GE5M2) against
the oracle: each kernel-A variant (X in TMEM, resident-X panel, streaming),
the logits and rounded gradient of forward_chunk, and the no-alloc entry."""
import numpy as np
import pytest
import torch

from synthetic import make_labels, make_W_f32, make_X, workload
from tests.gpu_common import need_gpu, run_step_with_operands, to_dev_i32, to_dev_u16, w_to_dev, w_to_host
from tests.parity import assert_operands_of_logits, assert_rel_close, assert_weights_close, check_step, positives

pytestmark = pytest.mark.gpu
DT = "fp8_ge5m2"


def _inputs(orc, w, step=0):
    X = make_X(w, step)
    rowptr, cols = make_labels(w, step)
    W = orc.sr_round(make_W_f32(w), "fp8", seed=0, step=2**64 - 1)      # E4M3 codes
    return W, X, rowptr, cols


CASES = [
    ("tiny", {"L": 1000, "d": 128, "B": 17}),             # X in TMEM, one M-block, ragged tail
    ("product3m_fp8", {"L": 2500, "B": 256}),             # X in TMEM, two M-blocks (the workload's shape)
    ("product3m_fp8", {"L": 900, "d": 1024, "B": 256}),   # resident-X panel (d > 768)
    ("tiny", {"L": 600, "d": 4096, "B": 64}),             # streaming kernel A (no panel fits)
]


@pytest.mark.parametrize("name,over", CASES)
def test_ge5m2_step_matches_oracle(orc, name, over):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload(name, dtype="fp8", **over)
    W, X, rowptr, cols = _inputs(orc, w)
    chunk = 512
    Wg, dXg, Zg, Gg = run_step_with_operands(elmo, W, X, rowptr, cols, w.lr, chunk, 0, 0, DT)
    r, _ = check_step(orc, W, X, rowptr, cols, w.lr, 0, 0, DT, Wg, dXg, Zg, Gg, chunk_rows=chunk)
    # and it is not the E4M3-gradient step: the operand grids differ
    r4 = orc.train_step(W, X, rowptr, cols, w.lr, 0, 0, "fp8")
    assert not np.array_equal(r["W"], r4["W"])


def test_ge5m2_forward_chunk_gradient_operand(orc):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("product3m_fp8", L=700, B=256)
    W, X, rowptr, cols = _inputs(orc, w)
    l0, l1 = 64, 700
    Wd = w_to_dev(W, "fp8")
    h = elmo.elmo_init_head(Wd, DT)
    Z = torch.empty(l1 - l0, w.B, device="cuda")
    G = torch.empty(l1 - l0, w.B, device="cuda")
    elmo.elmo_forward_chunk(h, to_dev_u16(X), to_dev_i32(rowptr), to_dev_i32(cols), l0, l1, Z, G)
    elmo.elmo_sync_status(h)
    r = orc.train_step(W, X, rowptr, cols, 0.0, 0, 0, DT, l0=l0, l1=l1, want_zg=True)
    assert_rel_close(Z.cpu().numpy(), r["Z"], "fp8", axis=None, what="Z")
    g, go, z = G.cpu().numpy(), r["G"], Z.cpu().numpy()
    # values on the E5M2 grid of 2^8 G, each the correctly rounded operand of its
    # own logit; equal to the oracle's where the logits agree
    codes = orc.rne_e5m2(g * 256.0)
    assert np.array_equal(orc.e5m2_value(codes) / 256.0, g)
    assert_operands_of_logits(g, z, positives(rowptr, cols, w.L, w.B, l0, l1), DT)
    same = z == r["Z"]
    assert np.array_equal(g[same], go[same])
    assert np.array_equal(w_to_host(Wd, "fp8"), W)
    h.close()


def test_ge5m2_noalloc_matches_head_step(orc):
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
    assert_weights_close(w_to_host(Wb, "fp8"), r["W"], "fp8", chunk_rows=1024)
    assert_rel_close(dXb.cpu().numpy(), r["dX"], DT, what="dX")
