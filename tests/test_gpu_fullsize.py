"""Parity at the full workload sizes, in the launch configuration bench.py uses
(label chunks of the workload), on outputs the oracle can compute one by one:
weight rows of sampled label ranges and dX rows of sampled samples (each a
function of its own row), and top-k rows of sampled queries."""
import numpy as np
import pytest
import torch

from synthetic import make_labels, make_X, workload
from tests.gpu_common import need_gpu, to_dev_i32, to_dev_u16, w_to_host
from tests.parity import (assert_operands_of_logits, assert_rel_close, assert_weights_close, flip_corrected_dx,
                           flip_corrected_weights)

pytestmark = pytest.mark.gpu


def _device_head(elmo, w):
    """W of the workload filled on the device by the library (Philox normal of
    std 0.02, stochastically rounded to the storage grid), as bench.py does;
    the oracle then starts from a host copy of exactly those weights."""
    Wd = torch.empty(w.L, w.d, dtype=torch.int16 if w.dtype == "bf16" else torch.uint8, device="cuda")
    return Wd, elmo.elmo_init_head(Wd, w.dtype, fill=True, init_std=0.02, seed=0)


def _label_ranges(L, chunk):
    # the first labels, a range straddling a chunk boundary, and the ragged tail
    mid = (L // chunk // 2) * chunk
    return [(0, 256), (max(0, mid - 128), mid + 128), (L - 300, L)]


@pytest.mark.parametrize("name", ["text500k_bf16", "product3m_fp8", "keyword8m6_bf16"])
def test_step_full_size_sampled(orc, name):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload(name)
    Wd, h = _device_head(elmo, w)
    W0 = w_to_host(Wd, w.dtype)
    X = make_X(w, 0)
    rowptr, cols = make_labels(w, 0)
    dX = torch.empty(w.B, w.d, device="cuda")
    samples = [0, w.B // 2, w.B - 1]
    Xd, rp, cl = to_dev_u16(X), to_dev_i32(rowptr), to_dev_i32(cols)
    if w.L <= 3_000_000:          # dX rows need every label; the 8.6M head checks weights only
        # logits and operands of the sampled samples over all labels, before the step
        Zs = np.empty((len(samples), w.L), np.float32)
        Gs = np.empty((len(samples), w.L), np.float32)
        for a in range(0, w.L, w.chunk):
            e = min(w.L, a + w.chunk)
            Zd = torch.empty(e - a, w.B, device="cuda")
            Gd = torch.empty(e - a, w.B, device="cuda")
            elmo.elmo_forward_chunk(h, Xd, rp, cl, a, e, Zd, Gd)
            Zs[:, a:e] = Zd[:, samples].T.cpu().numpy()
            Gs[:, a:e] = Gd[:, samples].T.cpu().numpy()
            del Zd, Gd
    # the operands of the checked label ranges before the step: where one of
    # them lands on the other neighbour of the oracle's (logits within rounding
    # of a midpoint), its label row is re-stepped from the GPU's operand
    ranges = _label_ranges(w.L, w.chunk)
    Granges = []
    for l0, l1 in ranges:
        Zd = torch.empty(l1 - l0, w.B, device="cuda")
        Gd = torch.empty(l1 - l0, w.B, device="cuda")
        elmo.elmo_forward_chunk(h, Xd, rp, cl, l0, l1, Zd, Gd)
        Granges.append(Gd.cpu().numpy())
    elmo.elmo_train_step_chunked(h, Xd, rp, cl, w.lr, w.chunk, 0, 0, dX)
    elmo.elmo_sync_status(h)
    for (l0, l1), Gg in zip(ranges, Granges):
        r = orc.train_step(W0[:l1], X, rowptr, cols, w.lr, 0, 0, w.dtype, l0=l0, l1=l1, want_dx=False, want_zg=True,
                           L=w.L)
        w_ref, _ = flip_corrected_weights(orc, W0, X, Gg, r["G"], r["W"], w.lr, 0, 0, w.dtype, l0=l0)
        assert_weights_close(w_to_host(Wd[l0:l1], w.dtype), w_ref, w.dtype)
    if w.L <= 3_000_000:
        ref, Zo, Go = orc.dx_rows(W0, X, rowptr, cols, samples, w.dtype, want_zg=True)
        Y = np.zeros((len(samples), w.L), np.float32)
        for i, b in enumerate(samples):
            Y[i, cols[rowptr[b]:rowptr[b + 1]]] = 1.0
        assert_rel_close(Zs, Zo, w.dtype, axis=None, what="Z rows")
        assert_operands_of_logits(Gs, Zs, Y, w.dtype, what="G rows (GPU)")
        assert_operands_of_logits(Go, Zo, Y, w.dtype, what="G rows (oracle)")
        dx_ref, _ = flip_corrected_dx(ref, Gs.T, Go.T, W0, w.dtype)
        assert_rel_close(dX.cpu().numpy()[samples], dx_ref, w.dtype, what="dX rows")
    h.close()


def test_topk_full_size_sampled(orc):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("topk5_3m_fp8")
    Wd = torch.empty(w.L, w.d, dtype=torch.uint8, device="cuda")
    h = elmo.elmo_init_head(Wd, "fp8", fill=True, init_std=0.02, seed=0)
    X = make_X(w, 0)
    idx = torch.empty(w.B, w.topk, dtype=torch.int32, device="cuda")
    sc = torch.empty(w.B, w.topk, device="cuda")
    elmo.elmo_topk_predict(h, to_dev_u16(X), w.topk, w.chunk, idx, sc)
    torch.cuda.synchronize()
    rows = [0, 511, 1023]
    ri, rs = orc.topk(w_to_host(Wd, "fp8"), X, w.topk, "fp8", rows=rows)
    assert np.array_equal(idx.cpu().numpy()[rows], ri)
    assert np.array_equal(sc.cpu().numpy()[rows].view(np.uint32), rs.view(np.uint32))
    h.close()
