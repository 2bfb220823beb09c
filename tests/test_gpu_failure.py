"""Failure detection on the GPU without a fault: a bounded wait that runs out
records ELMO_ETIMEOUT in the status word and the kernel returns, leaving the
context usable for the next step."""
import pytest
import torch

from synthetic import make_labels, make_W_bf16, make_X, workload
from tests.gpu_common import need_gpu, run_step
from tests.parity import assert_weights_close

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports_timeout(orc):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    status = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    elmo.elmo_check_bounded_wait(2_000_000, status)          # about 1 ms of clock
    torch.cuda.synchronize()
    assert status.cpu().tolist() == [4, elmo.WAIT_CHECK_SITE]  # ELMO_ETIMEOUT, the wait's site
    # the context still works: a step runs and matches the oracle
    w = workload("tiny", L=700, d=64, B=16)
    X = make_X(w, 0)
    rowptr, cols = make_labels(w, 0)
    W = make_W_bf16(w)
    Wg, _ = run_step(elmo, W, X, rowptr, cols, w.lr, 256, 0, 0, "bf16")
    r = orc.train_step(W, X, rowptr, cols, w.lr, 0, 0, "bf16")
    assert_weights_close(Wg, r["W"], "bf16")


def test_bounded_wait_rejects_bad_arguments():
    need_gpu()
    import precision_label_chunk_b200 as elmo
    lib = elmo.load()
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    assert lib.elmo_check_bounded_wait(0, status.data_ptr(), None) == 1          # ELMO_EINVAL
    assert lib.elmo_check_bounded_wait(2**33, status.data_ptr(), None) == 1
    assert lib.elmo_check_bounded_wait(1000, None, None) == 1
