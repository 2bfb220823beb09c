"""The persistent step kernel against the range-by-range kernels: the two
paths form the same gradient operands and draws, so the weights must agree
bit for bit (dX up to fp32 summation order), step after step."""
import os

import numpy as np
import pytest
import torch

from synthetic import make_labels, make_W_bf16, make_W_f32, make_X, workload
from tests.gpu_common import need_gpu, to_dev_i32, to_dev_u16, w_to_dev, w_to_host

pytestmark = pytest.mark.gpu


def _run(elmo, W, w, steps, fused, specials=None):
    os.environ["ELMO_STEP_FUSED"] = "1" if fused else "0"
    try:
        Wd = w_to_dev(W, w.dtype)
        h = elmo.elmo_init_head(Wd, w.dtype)
        dX = torch.empty(w.B, w.d, device="cuda")
        out = []
        for s in range(steps):
            X = to_dev_u16(make_X(w, s))
            rp, cl = make_labels(w, s)
            elmo.elmo_train_step_chunked(h, X, to_dev_i32(rp), to_dev_i32(cl), w.lr, 512, 0, s, dX)
            elmo.elmo_sync_status(h)
            out.append((w_to_host(Wd, w.dtype).copy(), dX.cpu().numpy().copy()))
        h.close()
        return out
    finally:
        os.environ.pop("ELMO_STEP_FUSED", None)


@pytest.mark.parametrize("dtype,L,d,B", [("bf16", 1200, 128, 32), ("bf16", 600, 128, 24), ("fp8", 1200, 128, 32),
                                         ("bf16", 700, 768, 256), ("fp8", 1000, 768, 256), ("bf16", 900, 256, 100),
                                         # rows of a partial 128-byte k-block (E4M3 d = 704: one 2-D box per
                                         # k-block) and a last ring stage past the k-blocks (bf16 d = 640)
                                         ("fp8", 900, 704, 256), ("bf16", 800, 640, 128),
                                         # bf16 with a last d-slice of 64 columns (one box in the W
                                         # slot the bulk store writes back)
                                         ("bf16", 700, 704, 64)])
def test_fused_step_matches_range_kernels(orc, dtype, L, d, B):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("tiny", dtype=dtype, L=L, d=d, B=B)
    W = make_W_bf16(w) if dtype == "bf16" else orc.sr_round(make_W_f32(w), "fp8", 0, 2**64 - 1)
    a = _run(elmo, W, w, 4, fused=False)
    b = _run(elmo, W, w, 4, fused=True)
    for s, ((wa, xa), (wb, xb)) in enumerate(zip(a, b)):
        bad = np.argwhere(wa != wb)
        assert bad.size == 0, (f"step {s}: {len(bad)} weights differ; rows {np.unique(bad[:, 0])[:20].tolist()}, "
                               f"cols {np.unique(bad[:, 1])[:20].tolist()}")
        assert np.allclose(xa, xb, rtol=1e-4, atol=1e-5), f"step {s}: dX differs"


def test_fused_step_special_weights(orc):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("tiny", dtype="bf16", L=600, d=128, B=24)
    W = make_W_bf16(w).copy()
    for i, c in enumerate([0x7F80, 0xFF80, 0x7FC0, 0x7F7F, 0xFF7F, 0x7F00, 0x0001, 0x8000]):
        W[3 + 70 * i, (13 * i) % w.d] = c
    a = _run(elmo, W, w, 1, fused=False)[0][0]
    b = _run(elmo, W, w, 1, fused=True)[0][0]
    bad = np.argwhere(a.view(np.uint16) != b.view(np.uint16))
    assert bad.size == 0, f"{len(bad)} weights differ: first {bad[:10].tolist()}"


@pytest.mark.parametrize("dtype,B,split", [("fp8", 256, "2"), ("fp8", 256, "140"), ("bf16", 128, "1"),
                                           ("bf16", 256, "142"), ("fp8", 96, "3")])
def test_fused_step_extreme_role_splits(orc, dtype, B, split, monkeypatch):
    """The dynamic tile queues and the ring under extreme splits of the SMs:
    one or two producer CTAs against all the rest, and almost every SM a
    producer (the split is clamped to leave one CTA per d-slice); the weights
    must not depend on it."""
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("tiny", dtype=dtype, L=20000, d=256, B=B)
    W = make_W_bf16(w) if dtype == "bf16" else orc.sr_round(make_W_f32(w), "fp8", 0, 2**64 - 1)
    a = _run(elmo, W, w, 2, fused=False)
    monkeypatch.setenv("ELMO_FUSED_A", split)
    b = _run(elmo, W, w, 2, fused=True)
    for s, ((wa, xa), (wb, xb)) in enumerate(zip(a, b)):
        assert np.array_equal(wa, wb), f"step {s}: {int((wa != wb).sum())} weights differ"
        # dX sums 20,000 labels' terms in an order that follows the split: fp32
        # reordering only, well inside 1e-4 of the rms
        rms = float(np.sqrt(np.mean(xb.astype(np.float64) ** 2)))
        assert np.allclose(xa, xb, rtol=1e-4, atol=1e-4 * rms), f"step {s}: dX differs"
