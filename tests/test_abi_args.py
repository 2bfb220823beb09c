"""Argument checking of the C ABI, on the host: every call below is rejected
before any CUDA work, so it runs without a GPU (device pointers are stand-in
addresses that are never dereferenced on the host)."""
import ctypes

import pytest

OK, EINVAL, EUNSUPPORTED = 0, 1, 5
DEV = 0x10000          # a 16-byte aligned stand-in device address


@pytest.fixture(scope="module")
def lib():
    import precision_label_chunk_b200 as elmo
    from precision_label_chunk_b200 import _build
    _build.build()
    return elmo.load()


def _err(lib):
    return lib.elmo_last_error().decode()


def test_init_head_shard_arguments(lib):
    out = ctypes.c_void_p()

    def init(W=DEV, L=1000, d=128, dt=1, base=0, total=1000, fill=0, std=0.02):
        return lib.elmo_init_head_shard(ctypes.byref(out), W, L, d, dt, base, total, fill, std, 0, None)

    assert init(W=None) == EINVAL
    assert init(dt=9) == EINVAL and "dtype" in _err(lib)
    assert init(dt=3, L=0) == EINVAL                                   # E5M2 heads take the same checks
    assert init(L=0) == EINVAL and init(L=1 << 24, total=1 << 24) == EINVAL
    assert init(base=-1) == EINVAL
    assert init(base=500, L=600, total=1000) == EINVAL and "outside a head" in _err(lib)
    assert init(total=(1 << 31), L=1000, base=0) == EINVAL             # label ids are int32
    assert init(d=100) == EINVAL and init(d=8192) == EINVAL
    assert init(W=DEV + 8) == EINVAL and "aligned" in _err(lib)
    assert init(fill=1, std=-1.0) == EINVAL
    assert not out.value                                               # no head was made


def test_topk_merge_arguments(lib):
    m = lambda P=2, B=4, k=5, p=DEV: lib.elmo_topk_merge(p, DEV, P, B, k, DEV, DEV, None)   # noqa: E731
    assert m(p=None) == EINVAL
    assert m(P=0) == EINVAL and m(P=65) == EINVAL
    assert m(B=0) == EINVAL and m(B=4097) == EINVAL
    assert m(k=0) == EINVAL and m(k=65) == EINVAL


def test_elementwise_calls_arguments(lib):
    assert lib.elmo_kahan_sgd(DEV, DEV, DEV, -1, 0.1, None) == EINVAL
    assert lib.elmo_kahan_sgd(None, DEV, DEV, 5, 0.1, None) == EINVAL
    assert lib.elmo_kahan_sgd(DEV, DEV, DEV, 5, float("inf"), None) == EINVAL
    assert lib.elmo_kahan_sgd(None, None, None, 0, 0.1, None) == OK        # n = 0: nothing to do
    assert lib.elmo_round_bf16(DEV, DEV, -1, None) == EINVAL
    assert lib.elmo_round_bf16(None, DEV, 3, None) == EINVAL
    assert lib.elmo_round_bf16(None, None, 0, None) == OK
    assert lib.elmo_sr_round(DEV, DEV, 8, 2, 0, 0, 0, None) == EINVAL       # the E5M2-gradient head dtype is no grid
    assert lib.elmo_sr_round(DEV, DEV, 8, 7, 0, 0, 0, None) == EINVAL
    assert lib.elmo_sr_round(DEV, DEV, 16, 1, 0, 0, 2**64 - 8, None) == EINVAL   # indices would wrap
    assert lib.elmo_sr_round(None, None, 0, 3, 0, 0, 0, None) == OK
    assert lib.elmo_sr_draws(DEV, -1, 0, 0, 0, None) == EINVAL


def test_metric_and_check_arguments(lib):
    p = lambda B=4, k=5, nnz=3, i=DEV: lib.elmo_precision_at_k(i, B, k, DEV, DEV, nnz, DEV, None)   # noqa: E731
    assert p(i=None) == EINVAL
    assert p(B=0) == EINVAL and p(k=65) == EINVAL and p(nnz=-1) == EINVAL
    assert lib.elmo_check_bounded_wait(1000, None, None) == EINVAL
    assert lib.elmo_check_bounded_wait(0, DEV, None) == EINVAL
    assert lib.elmo_check_bounded_wait((1 << 32) + 1, DEV, None) == EINVAL


def test_calls_on_a_null_head(lib):
    n = ctypes.c_int64()
    t = ctypes.c_double()
    assert lib.elmo_launch_count(None, ctypes.byref(n)) == EINVAL
    assert lib.elmo_profile_enable(None, 1) == EINVAL
    assert lib.elmo_profile_read(None, 0, ctypes.byref(t), ctypes.byref(n)) == EINVAL
    assert lib.elmo_sync_status(None, None) == EINVAL
    assert lib.elmo_train_step_chunked(None, DEV, 4, DEV, DEV, 3, 0.1, 128, 0, 0, DEV, None) == EINVAL
    assert lib.elmo_topk_predict(None, DEV, 4, 5, 128, DEV, DEV, None) == EINVAL
    assert lib.elmo_head_destroy(None) == OK
