"""Kahan-compensated SGD and the bf16 hand-off of dX on the GPU against the
oracle: bit-exact (both are sequences of IEEE fp32 operations and one
rounding to nearest-even per stored value)."""
import numpy as np
import pytest
import torch

from tests.gpu_common import need_gpu

pytestmark = pytest.mark.gpu


def _bf16(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _specials():
    return np.array([0.0, -0.0, np.inf, -np.inf, np.nan, 1e-40, -1e-39, 3.0e38, -3.3e38, 1.0, 2.0**-133],
                    np.float32)


def _state(rng, n):
    p = _bf16(rng.standard_normal(n) * 0.05)
    c = _bf16(rng.standard_normal(n) * 1e-4)
    g = _bf16(rng.standard_normal(n))
    sp = _bf16(_specials())
    m = min(n, sp.size)
    p[:m], c[n - m:], g[:m] = sp[:m], sp[:m], np.roll(sp[:m], 3)
    return p, c, g


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


@pytest.mark.parametrize("n,offset", [(1, 0), (7, 0), (8, 0), (4096 + 5, 0), (100_003, 1), (1 << 20, 0), (0, 0)])
def test_kahan_sgd_matches_oracle(orc, n, offset):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    rng = np.random.default_rng(n + offset)
    p, c, g = _state(rng, max(n, 1))
    p, c, g = p[:n], c[:n], g[:n]
    # offset 1: the buffers start 2 bytes past a 16-byte boundary (scalar path)
    P = _dev(np.concatenate([np.zeros(offset, np.uint16), p]))[offset:]
    C = _dev(np.concatenate([np.zeros(offset, np.uint16), c]))[offset:]
    G = _dev(np.concatenate([np.zeros(offset, np.uint16), g]))[offset:]
    lr = 0.0123
    elmo.elmo_kahan_sgd(P, C, G, lr)
    torch.cuda.synchronize()
    wp, wc = orc.kahan_sgd(p, c, g, lr)
    assert np.array_equal(P.cpu().numpy().view(np.uint16), wp)
    assert np.array_equal(C.cpu().numpy().view(np.uint16), wc)


def test_kahan_sgd_trajectory_matches_oracle(orc):
    """Fifty steps, each side on its own state, with fresh gradients."""
    need_gpu()
    import precision_label_chunk_b200 as elmo
    rng = np.random.default_rng(7)
    n = 50_000
    p = _bf16(1.0 + rng.random(n))
    c = np.zeros(n, np.uint16)
    P, C = _dev(p), _dev(c)
    for s in range(50):
        g = _bf16(1.0 + 0.5 * rng.standard_normal(n))
        elmo.elmo_kahan_sgd(P, C, _dev(g), 1e-4)
        p, c = orc.kahan_sgd(p, c, g, 1e-4)
    torch.cuda.synchronize()
    assert np.array_equal(P.cpu().numpy().view(np.uint16), p)
    assert np.array_equal(C.cpu().numpy().view(np.uint16), c)


def test_kahan_sgd_full_size_sampled(orc):
    """The benchmark's size (110M parameters): every element is independent, so
    a sample of positions checked against the oracle on those positions alone."""
    need_gpu()
    import precision_label_chunk_b200 as elmo
    n = 110_000_000
    gen = torch.Generator(device="cuda")
    gen.manual_seed(3)
    P = (torch.randn(n, generator=gen, device="cuda") * 0.05).to(torch.bfloat16)
    C = (torch.randn(n, generator=gen, device="cuda") * 1e-4).to(torch.bfloat16)
    G = torch.randn(n, generator=gen, device="cuda").to(torch.bfloat16)
    pos = torch.from_numpy(np.unique(np.concatenate([np.random.default_rng(4).integers(0, n, 20000),
                                                     np.arange(n - 9, n)]))).cuda()
    p0, c0, g0 = (t[pos].view(torch.int16).cpu().numpy().view(np.uint16) for t in (P, C, G))
    elmo.elmo_kahan_sgd(P, C, G, 0.02)
    torch.cuda.synchronize()
    wp, wc = orc.kahan_sgd(p0, c0, g0, 0.02)
    assert np.array_equal(P[pos].view(torch.int16).cpu().numpy().view(np.uint16), wp)
    assert np.array_equal(C[pos].view(torch.int16).cpu().numpy().view(np.uint16), wc)


@pytest.mark.parametrize("n,offset", [(1, 0), (9, 0), (256 * 768, 0), (1000, 1), (0, 0)])
def test_round_bf16_matches_oracle(orc, n, offset):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    rng = np.random.default_rng(n)
    with np.errstate(over="ignore"):                         # magnitudes past fp32's range become +-inf
        x = (rng.standard_normal(max(n, 1)) * 10.0 ** rng.integers(-45, 39, max(n, 1))).astype(np.float32)[:n]
    # exact ties between bf16 neighbours (round to even either way)
    t = (_bf16_pattern_ties(min(n, 64)))
    x[:t.size] = t
    sp = _specials()
    x[-min(n, sp.size):] = sp[:min(n, sp.size)] if n else x[:0]
    X = torch.from_numpy(np.concatenate([np.zeros(offset, np.float32), x])).cuda()[offset:]
    out = torch.empty(n + offset, dtype=torch.int16, device="cuda")[offset:]
    elmo.elmo_round_bf16(X, out)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().view(np.uint16), orc.rne_bf16(x))


def _bf16_pattern_ties(m):
    """fp32 values exactly halfway between two bf16 neighbours."""
    base = np.arange(m, dtype=np.uint32) * 0x00530000 + 0x3F800000
    return (base | 0x8000).view(np.float32)
