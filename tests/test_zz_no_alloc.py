"""The allocation-free training step gives what the head-based step gives.

elmo_train_step_noalloc is for callers that cannot allocate device memory
(code issuing the step during CUDA-graph stream capture, runtimes with a fixed
memory budget): it keeps all of its scratch in one static device array.  This
file is collected last on purpose, so that a run stopping at the first failure
has already run every other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from synthetic import make_labels, make_W_f32, make_W_bf16, make_X, workload
from tests.gpu_common import need_gpu, to_dev_i32, to_dev_u16, w_to_dev, w_to_host
from tests.parity import assert_rel_close

pytestmark = pytest.mark.gpu


def _start_weights(orc, w):
    if w.dtype == "bf16":
        return make_W_bf16(w)
    return orc.sr_round(make_W_f32(w), "fp8", seed=0, step=2**64 - 1)


@pytest.mark.parametrize("name,over", [("product3m_fp8", {"L": 70_000, "B": 256}),
                                       ("text500k_bf16", {"L": 40_000, "B": 200})])
def test_noalloc_step_matches_head_step_twice(orc, name, over):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload(name, **over)
    W0 = _start_weights(orc, w)
    W_head, W_free = w_to_dev(W0, w.dtype), w_to_dev(W0, w.dtype)
    head = elmo.elmo_init_head(W_head, w.dtype)
    dX_head = torch.empty(w.B, w.d, device="cuda")
    dX_free = torch.empty(w.B, w.d, device="cuda")
    status = torch.full((2,), 7, dtype=torch.int32, device="cuda")
    for step in (0, 1):                        # two calls in a row share the static scratch
        X = to_dev_u16(make_X(w, step))
        rowptr, cols = (to_dev_i32(a) for a in make_labels(w, step))
        elmo.elmo_train_step_chunked(head, X, rowptr, cols, w.lr, w.chunk, 5, step, dX_head)
        elmo.elmo_train_step_noalloc(W_free, w.dtype, X, rowptr, cols, w.lr, w.chunk, 5, step, dX_free, status)
        elmo.elmo_sync_status(head)
        torch.cuda.synchronize()
        assert status.cpu().tolist() == [0, 0]
        # the same kernels and the same index-keyed draws: the weights agree bit for bit,
        # even though this path splits a chunk into shorter passes to fit its fixed scratch
        assert torch.equal(W_free, W_head), f"step {step}: weights differ from the head-based step"
        assert_rel_close(dX_free.cpu().numpy(), dX_head.cpu().numpy(), w.dtype, what=f"dX step {step}")
    head.close()


def test_noalloc_rejects_sizes_beyond_its_limits():
    need_gpu()
    import precision_label_chunk_b200 as elmo
    W = torch.zeros(1024, 64, dtype=torch.bfloat16, device="cuda")
    X = torch.zeros(300, 64, dtype=torch.bfloat16, device="cuda")          # B above 256
    rowptr = torch.zeros(301, dtype=torch.int32, device="cuda")
    cols = torch.zeros(0, dtype=torch.int32, device="cuda")
    dX = torch.empty(300, 64, device="cuda")
    status = torch.zeros(2, dtype=torch.int32, device="cuda")
    with pytest.raises(elmo.ElmoError) as ei:
        elmo.elmo_train_step_noalloc(W, "bf16", X, rowptr, cols, 0.1, 512, 0, 0, dX, status)
    assert ei.value.status == 5 and "B = 300" in str(ei.value)
