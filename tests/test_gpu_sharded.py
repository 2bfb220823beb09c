"""A head split by labels, run shard by shard on one GPU (no kernel of one
shard waits on another): the shards' rows equal the unsplit head's bit for
bit, their input gradients add up to its dX, and the merged top-k equals its
top-k; both sides also against the oracle."""
import numpy as np
import pytest
import torch

from synthetic import make_labels, make_W_bf16, make_W_f32, make_X, workload
from tests.gpu_common import need_gpu, to_dev_i32, to_dev_u16, w_to_dev, w_to_host
from tests.parity import assert_rel_close, assert_weights_close

pytestmark = pytest.mark.gpu

# shard boundaries: tile-aligned, unaligned, and a one-row shard
SPLITS = [[0, 384, 1000], [0, 300, 301, 1000], [0, 1000]]


def _inputs(orc, w, step=0):
    X = make_X(w, step)
    rowptr, cols = make_labels(w, step)
    W = make_W_bf16(w) if w.dtype == "bf16" else orc.sr_round(make_W_f32(w), "fp8", seed=0, step=2**64 - 1)
    return W, X, rowptr, cols


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("bounds", SPLITS)
def test_sharded_fill_matches_whole_head(dtype, bounds):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    L, d = bounds[-1], 128
    wdt = torch.int16 if dtype == "bf16" else torch.uint8
    Wfull = torch.empty(L, d, dtype=wdt, device="cuda")
    elmo.elmo_init_head(Wfull, dtype, fill=True, init_std=0.02, seed=5).close()
    parts = []
    for a, b in zip(bounds[:-1], bounds[1:]):
        Ws = torch.empty(b - a, d, dtype=wdt, device="cuda")
        elmo.elmo_init_head_shard(Ws, a, L, dtype, fill=True, init_std=0.02, seed=5).close()
        parts.append(Ws)
    assert torch.equal(torch.cat(parts), Wfull)


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("bounds", SPLITS)
def test_sharded_step_matches_whole_head(orc, dtype, bounds):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("tiny", dtype=dtype, L=bounds[-1], d=128, B=40, lam=30)
    W, X, rowptr, cols = _inputs(orc, w)
    Xd, rp, cl = to_dev_u16(X), to_dev_i32(rowptr), to_dev_i32(cols)
    chunk = 256
    # the whole head
    Wd = w_to_dev(W, dtype)
    h = elmo.elmo_init_head(Wd, dtype)
    dX = torch.empty(w.B, w.d, device="cuda")
    elmo.elmo_train_step_chunked(h, Xd, rp, cl, w.lr, chunk, 3, 7, dX)
    elmo.elmo_sync_status(h)                           # raises on a nonzero status
    h.close()
    # the same step, shard by shard, with the whole head's labels
    parts, dX_sum = [], torch.zeros(w.B, w.d, device="cuda")
    for a, b in zip(bounds[:-1], bounds[1:]):
        Ws = w_to_dev(W[a:b], dtype)
        hs = elmo.elmo_init_head_shard(Ws, a, w.L, dtype)
        dXs = torch.empty(w.B, w.d, device="cuda")
        elmo.elmo_train_step_chunked(hs, Xd, rp, cl, w.lr, chunk, 3, 7, dXs)
        elmo.elmo_sync_status(hs)                      # other shards' labels are not errors
        hs.close()
        parts.append(w_to_host(Ws, dtype))
        dX_sum += dXs
    assert np.array_equal(np.concatenate(parts), w_to_host(Wd, dtype))
    # dX: the same terms summed in another order
    ref = dX.cpu().numpy()
    np.testing.assert_allclose(dX_sum.cpu().numpy(), ref, rtol=1e-4, atol=1e-5 * float(np.abs(ref).max()))
    # and the oracle's step of the whole head
    r = orc.train_step(W, X, rowptr, cols, w.lr, 3, 7, dtype)
    assert_weights_close(np.concatenate(parts), r["W"], dtype, chunk_rows=chunk)
    assert_rel_close(dX_sum.cpu().numpy(), r["dX"], dtype, what="dX")


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_shard_rejects_labels_outside_the_whole_head(dtype):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    L, d, B = 1000, 128, 4
    wdt = torch.int16 if dtype == "bf16" else torch.uint8
    Ws = torch.zeros(200, d, dtype=wdt, device="cuda")
    hs = elmo.elmo_init_head_shard(Ws, 500, L, dtype)
    X = torch.zeros(B, d, dtype=torch.int16, device="cuda")
    dX = torch.empty(B, d, device="cuda")
    rp = to_dev_i32([0, 1, 2, 3, 4])
    ok = to_dev_i32([0, 499, 700, 999])                # below, inside, beyond the shard: all valid
    elmo.elmo_train_step_chunked(hs, X, rp, ok, 0.1, 128, 0, 0, dX)
    elmo.elmo_sync_status(hs)                          # raises on a nonzero status
    bad = to_dev_i32([0, 600, 1000, 5])                # 1000 is outside the whole head
    elmo.elmo_train_step_chunked(hs, X, rp, bad, 0.1, 128, 0, 0, dX)
    with pytest.raises(elmo.ElmoError) as ei:
        elmo.elmo_sync_status(hs)
    assert ei.value.status == 6                        # ELMO_EDATA
    hs.close()
    with pytest.raises(elmo.ElmoError):
        elmo.elmo_init_head_shard(Ws, 900, L, dtype)   # rows [900, 1100) outside 1000 labels


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("bounds", [[0, 4096, 8192, 9000], [0, 3000, 3001, 6000]])
def test_sharded_topk_merge_matches_whole_head(orc, dtype, bounds):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    L, k = bounds[-1], 7
    w = workload("tiny", dtype=dtype, L=L, d=128, B=300)
    W, X, _, _ = _inputs(orc, w)
    Xd = to_dev_u16(X)
    idx = torch.empty(w.B, k, dtype=torch.int32, device="cuda")
    sc = torch.empty(w.B, k, dtype=torch.float32, device="cuda")
    h = elmo.elmo_init_head(w_to_dev(W, dtype), dtype)
    elmo.elmo_topk_predict(h, Xd, k, 2048, idx, sc)
    h.close()
    P = len(bounds) - 1
    gi = torch.empty(P, w.B, k, dtype=torch.int32, device="cuda")
    gs = torch.empty(P, w.B, k, dtype=torch.float32, device="cuda")
    for p, (a, b) in enumerate(zip(bounds[:-1], bounds[1:])):
        kk = min(k, b - a)
        if kk < k:                                      # a one-row shard: pad its list with ranked-last entries
            gi[p].fill_(2**31 - 1)
            gs[p].fill_(float("nan"))
        hs = elmo.elmo_init_head_shard(w_to_dev(W[a:b], dtype), a, L, dtype)
        li = torch.empty(w.B, kk, dtype=torch.int32, device="cuda")
        ls = torch.empty(w.B, kk, dtype=torch.float32, device="cuda")
        elmo.elmo_topk_predict(hs, Xd, kk, 2048, li, ls)
        hs.close()
        gi[p, :, :kk] = li
        gs[p, :, :kk] = ls
        assert int(li.min()) >= a and int(li.max()) < b   # label ids of the whole head
    mi = torch.empty_like(idx)
    ms = torch.empty_like(sc)
    elmo.elmo_topk_merge(gi, gs, mi, ms)
    torch.cuda.synchronize()
    assert torch.equal(mi, idx)
    assert torch.equal(ms.view(torch.int32), sc.view(torch.int32))
    rows = np.arange(0, w.B, 37)
    oi, os_ = orc.topk(W, X, k, dtype, rows=rows)
    assert np.array_equal(mi.cpu().numpy()[rows], oi)
    assert np.array_equal(ms.cpu().numpy()[rows].view(np.int32), os_.view(np.int32))


def test_topk_merge_order_rules():
    """Lists built on the host with ties, signed zeros, infinities and NaN; the
    merge must give the union's best k in the ranking order (score descending,
    NaN last, ties to the lower label id)."""
    need_gpu()
    import precision_label_chunk_b200 as elmo
    rng = np.random.default_rng(11)
    P, B, k = 5, 64, 9
    vals = np.array([1.5, 1.5, 0.0, -0.0, np.inf, -np.inf, np.nan, 2.0, -3.0, 1e-30], np.float32)
    ids = rng.permutation(P * B * k * 4)[: P * B * k].astype(np.int32).reshape(P, B, k)
    sc = vals[rng.integers(0, len(vals), size=(P, B, k))]
    sc = np.where(rng.random((P, B, k)) < 0.5, rng.standard_normal((P, B, k)).astype(np.float32), sc)

    def key(s, i):
        return (1, 0.0, i) if np.isnan(s) else (0, -float(s), i)

    for p in range(P):                      # each list sorted best first
        for b in range(B):
            order = sorted(range(k), key=lambda j: key(sc[p, b, j], ids[p, b, j]))
            sc[p, b] = sc[p, b, order]
            ids[p, b] = ids[p, b, order]
    want_i = np.zeros((B, k), np.int32)
    want_s = np.zeros((B, k), np.float32)
    for b in range(B):
        pool = sorted(((sc[p, b, j], ids[p, b, j]) for p in range(P) for j in range(k)), key=lambda t: key(*t))
        want_s[b] = [t[0] for t in pool[:k]]
        want_i[b] = [t[1] for t in pool[:k]]
    gi, gs = torch.from_numpy(ids).cuda(), torch.from_numpy(sc).cuda()
    mi = torch.empty(B, k, dtype=torch.int32, device="cuda")
    ms = torch.empty(B, k, dtype=torch.float32, device="cuda")
    elmo.elmo_topk_merge(gi, gs, mi, ms)
    torch.cuda.synchronize()
    assert np.array_equal(mi.cpu().numpy(), want_i)
    got = ms.cpu().numpy()
    assert np.array_equal(np.isnan(got), np.isnan(want_s))
    assert np.array_equal(got[~np.isnan(got)].view(np.int32), want_s[~np.isnan(want_s)].view(np.int32))
