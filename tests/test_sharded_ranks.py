"""The label split of the head on CPU: the shard ranges, and (gloo, world size
2) the reduction of the ranks' input gradients and the gathering of their top-k
lists, alone and through ShardedHead.  Each rank's share of the step is
computed by the oracle over its label rows (the GPU kernels are not involved);
the sum over ranks must be the oracle's step of the whole head."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("world", [1, 2, 3, 8])
@pytest.mark.parametrize("L", [1024, 1025, 4096 + 77, 3_000_000, 2**24 + 5])
def test_label_shard_partitions_the_head(L, world):
    sys.path.insert(0, ROOT)
    from precision_label_chunk_b200.sharded import label_shard
    shards = [label_shard(L, r, world) for r in range(world)]
    assert shards[0][0] == 0
    for (a, n), (b, _) in zip(shards, shards[1:]):
        assert a + n == b                                   # contiguous, no gap, no overlap
    assert shards[-1][0] + shards[-1][1] == L
    assert all(n >= 1 for _, n in shards)
    assert all(a % 128 == 0 for a, _ in shards)             # boundaries on tile boundaries
    sizes = [n for _, n in shards[:-1]] + [-(-shards[-1][1] // 128) * 128]
    assert max(sizes) - min(sizes) <= 128                   # balanced to a tile


def test_label_shard_needs_a_tile_per_rank():
    sys.path.insert(0, ROOT)
    from precision_label_chunk_b200.sharded import label_shard
    with pytest.raises(ValueError):
        label_shard(200, 0, 3)
    with pytest.raises(ValueError):
        label_shard(1000, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(dtype):
    import oracle
    from synthetic import make_labels, make_W_bf16, make_W_f32, make_X, workload
    w = workload("tiny", dtype=dtype, L=1100, d=64, B=24, lam=20)
    W = make_W_bf16(w) if dtype == "bf16" else oracle.sr_round(make_W_f32(w), "fp8", seed=0, step=2**64 - 1)
    X = make_X(w, 0)
    rowptr, cols = make_labels(w, 0)
    return w, W, X, rowptr, cols


def _rank_main(rank, world, port, dtype, out):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from precision_label_chunk_b200.sharded import gather_topk, label_shard, reduce_input_grad
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    w, W, X, rowptr, cols = _inputs(dtype)
    a, n = label_shard(w.L, rank, world)
    r = oracle.train_step(W, X, rowptr, cols, w.lr, 9, 4, dtype, l0=a, l1=a + n, nthreads=1)
    dX = torch.from_numpy(r["dX"].copy())
    reduce_input_grad(dX)
    idx, sc = oracle.topk(W[a:a + n], X, 6, dtype, nthreads=1)
    gi, gs = gather_topk(torch.from_numpy(idx + a), torch.from_numpy(sc))
    out.put((rank, a, r["W"], dX.numpy(), gi.numpy(), gs.numpy()))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_split_step_sums_to_whole_head_gloo(orc, dtype):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, dtype, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w, W, X, rowptr, cols = _inputs(dtype)
    whole = orc.train_step(W, X, rowptr, cols, w.lr, 9, 4, dtype, nthreads=1)
    # rows: the SR of a label's row depends on nothing but that row's step
    assert np.array_equal(np.concatenate([t[2] for t in res]), whole["W"])
    # dX: each rank's labels summed on that rank, then across ranks
    ref = whole["dX"]
    for t in res:
        np.testing.assert_allclose(t[3], ref, rtol=1e-5, atol=1e-6 * float(np.abs(ref).max()))
        assert np.array_equal(t[3], res[0][3])              # every rank holds the same sum
    # top-k: the best 6 of the union of the ranks' lists is the whole head's top-6
    gi, gs = res[0][4], res[0][5]
    assert gi.shape == (world, w.B, 6)
    oi, osc = orc.topk(W, X, 6, dtype, nthreads=1)
    for b in range(w.B):
        pool = sorted(zip(gs[:, b].ravel().tolist(), gi[:, b].ravel().tolist()), key=lambda t: (-t[0], t[1]))
        assert [i for _, i in pool[:6]] == oi[b].tolist()


def _class_rank_main(rank, world, port, dtype, out):
    """ShardedHead itself over gloo: the library calls it makes are stood in
    for by the oracle on this rank's rows (test only), so that its plumbing
    (shard rows, label ids of the whole head, the dX reduction, the gather
    and merge of the top-k lists) runs as in a multi-GPU job."""
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from precision_label_chunk_b200 import sharded
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    w, W, X, rowptr, cols = _inputs(dtype)

    class FakeHead:
        def __init__(self, Wl, base, total):
            self.W, self.base, self.total = Wl, base, total

    def init_shard(Wl, base, total, *a, **k):
        return FakeHead(Wl, base, total)

    def train_step(h, Xt, rp, cl, lr, chunk, seed, step, dX, stream=None):
        n = h.W.shape[0]
        Wfull = np.zeros((h.total, w.d), h.W.numpy().dtype)
        Wfull[h.base:h.base + n] = h.W.numpy()
        r = oracle.train_step(Wfull, Xt.numpy(), rp.numpy(), cl.numpy(), lr, seed, step, dtype,
                              l0=h.base, l1=h.base + n, nthreads=1)
        h.W.copy_(torch.from_numpy(r["W"]))
        dX.copy_(torch.from_numpy(r["dX"]))

    def topk_predict(h, Xt, k, chunk, idx, score, stream=None):
        i, s = oracle.topk(h.W.numpy(), Xt.numpy(), k, dtype, nthreads=1)
        idx.copy_(torch.from_numpy(i + h.base))
        score.copy_(torch.from_numpy(s))

    def topk_merge(gi, gs, idx, score, stream=None):
        P, B, k = gi.shape
        for b in range(B):
            pool = sorted(zip(gs[:, b].reshape(-1).tolist(), gi[:, b].reshape(-1).tolist()), key=lambda t: (-t[0], t[1]))
            idx[b] = torch.tensor([t[1] for t in pool[:k]], dtype=idx.dtype)
            score[b] = torch.tensor([t[0] for t in pool[:k]], dtype=score.dtype)

    sharded.elmo_init_head_shard = init_shard
    sharded.elmo_train_step_chunked = train_step
    sharded.elmo_topk_predict = topk_predict
    sharded.elmo_topk_merge = topk_merge
    base, rows = sharded.label_shard(w.L, rank, world)
    Wl = torch.from_numpy(W[base:base + rows].copy())
    head = sharded.ShardedHead(Wl, w.L, dtype)
    dX = torch.zeros(w.B, w.d)
    head.train_step(torch.from_numpy(X), torch.from_numpy(rowptr), torch.from_numpy(cols), w.lr, 512, 9, 4, dX)
    idx = torch.zeros(w.B, 6, dtype=torch.int32)
    sc = torch.zeros(w.B, 6)
    head.topk_predict(torch.from_numpy(X), 6, 512, idx, sc)
    out.put((rank, head.label_base, Wl.numpy(), dX.numpy(), idx.numpy(), sc.numpy()))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("dtype", ["fp8"])
def test_sharded_head_class_over_gloo(orc, dtype):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_class_rank_main, args=(r, world, port, dtype, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w, W, X, rowptr, cols = _inputs(dtype)
    whole = orc.train_step(W, X, rowptr, cols, w.lr, 9, 4, dtype, nthreads=1)
    assert [t[1] for t in res] == [0, res[1][1]] and res[1][1] % 128 == 0
    assert np.array_equal(np.concatenate([t[2] for t in res]), whole["W"])      # updated in place, rank by rank
    ref = whole["dX"]
    for t in res:
        np.testing.assert_allclose(t[3], ref, rtol=1e-5, atol=1e-6 * float(np.abs(ref).max()))
    # the top-k of the updated head: every rank holds the same merged lists
    oi, osc = orc.topk(whole["W"], X, 6, dtype, nthreads=1)
    for t in res:
        assert np.array_equal(t[4], oi)
        assert np.array_equal(t[5].view(np.int32), osc.view(np.int32))
