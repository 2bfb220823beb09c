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
