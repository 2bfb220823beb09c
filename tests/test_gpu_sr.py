"""GPU stochastic rounding and its random draws are bit-exact with the oracle."""
import ctypes

import numpy as np
import pytest
import torch

from tests.gpu_common import need_gpu

pytestmark = pytest.mark.gpu


def _adversarial(dtype, rng):
    import ml_dtypes
    if dtype == "bf16":
        g = np.arange(0, 0x7F80, dtype=np.uint16).view(ml_dtypes.bfloat16).astype(np.float32)
        step = np.abs(np.diff(g.astype(np.float64)))
        mids = (g[:-1].astype(np.float64) + step / 2).astype(np.float32)
    elif dtype == "e5m2":
        g = np.arange(0, 0x7C, dtype=np.uint8).view(ml_dtypes.float8_e5m2).astype(np.float32)
        mids = ((g[:-1].astype(np.float64) + g[1:]) / 2).astype(np.float32)
    else:
        g = np.arange(0, 127, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float32)
        mids = ((g[:-1].astype(np.float64) + g[1:]) / 2).astype(np.float32)
    near = np.concatenate([np.nextafter(g, np.float32(np.inf)), np.nextafter(g, np.float32(0))])
    special = np.array([0.0, -0.0, np.inf, -np.inf, np.nan, 448.0, 447.99, 448.01, 480.0, 1e30, 3.4e38,
                        3.3895313892515355e38, 1e-45, -1e-45, 1e-39, 2.0 ** -10, 2.0 ** -9, 2.0 ** -6,
                        2.0 ** -7 + 2.0 ** -12, 57344.0, 57343.99, 57345.0, 61440.0, 2.0 ** -16, 2.0 ** -17,
                        2.0 ** -14, 2.0 ** -14 + 2.0 ** -30, 2.0 ** -14 - 2.0 ** -30, 3 * 2.0 ** -18], np.float32)
    x = np.concatenate([g, mids, near, special])
    x = np.concatenate([x, -x])
    rnd = (rng.standard_normal(1 << 20) * 0.05).astype(np.float32)
    wide = (rng.random(1 << 18) * 2 - 1).astype(np.float32) * np.exp2(rng.integers(-140, 120, 1 << 18)).astype(np.float32)
    return np.concatenate([x, rnd, wide]).astype(np.float32)


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "e5m2"])
@pytest.mark.parametrize("seed,step,base", [(0, 0, 0), (0xDEADBEEF12345678, 2**63 + 5, 13), (7, 2**64 - 1, 2**40 + 3)])
def test_sr_round_bit_exact(orc, dtype, seed, step, base):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    x = _adversarial(dtype, np.random.default_rng(seed & 0xFFFF))
    ref = orc.sr_round(x, dtype, seed, step, base)
    xd = torch.from_numpy(x).cuda()
    out = torch.empty(x.size, dtype=torch.int16 if dtype == "bf16" else torch.uint8, device="cuda")
    elmo.elmo_sr_round(xd, out, dtype, seed, step, base)
    got = out.cpu().numpy().view(np.uint16 if dtype == "bf16" else np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first x={x[bad[:5]]} got={got[bad[:5]]} ref={ref[bad[:5]]}"


def test_sr_round_large_random_bit_exact(orc):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    rng = np.random.default_rng(99)
    x = (rng.standard_normal(10_000_000) * 0.03).astype(np.float32)
    for dtype in ("bf16", "fp8", "e5m2"):
        ref = orc.sr_round(x, dtype, 3, 11, 5)
        out = torch.empty(x.size, dtype=torch.int16 if dtype == "bf16" else torch.uint8, device="cuda")
        elmo.elmo_sr_round(torch.from_numpy(x).cuda(), out, dtype, 3, 11, 5)
        got = out.cpu().numpy().view(np.uint16 if dtype == "bf16" else np.uint8)
        assert np.array_equal(got, ref)


@pytest.mark.parametrize("dtype", ["bf16", "fp8", "e5m2"])
@pytest.mark.parametrize("base,off,tail", [(8, 0, 5), (2**35, 0, 0), (0, 1, 3), (16, 4, 7), (2**60 + 8, 0, 1)])
def test_sr_round_whole_blocks_and_tails(orc, dtype, base, off, tail):
    """Whole 8-value blocks at 8-aligned indices and 16-byte aligned buffers take
    the vectorised kernel; a ragged tail, an unaligned index base or a buffer
    that starts off a 16-byte boundary take the per-value kernel: all must give
    the oracle's codes."""
    need_gpu()
    import precision_label_chunk_b200 as elmo
    x = _adversarial(dtype, np.random.default_rng(base & 0xFFFF))
    n = ((x.size - off) // 8) * 8 - 8 + tail
    ref = orc.sr_round(x[off:off + n], dtype, 21, 4, base)
    xd = torch.from_numpy(x).cuda()[off:off + n]          # off > 0: the input starts 4*off bytes past alignment
    odt = torch.int16 if dtype == "bf16" else torch.uint8
    out_full = torch.empty(n + off, dtype=odt, device="cuda")
    out = out_full[off:]
    elmo.elmo_sr_round(xd, out, dtype, 21, 4, base)
    got = out.cpu().numpy().view(np.uint16 if dtype == "bf16" else np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first at {bad[:5]}"


@pytest.mark.parametrize("seed,step,base,n", [(0, 0, 0, 1000), (5, 9, 3, 4097), (2**64 - 1, 2**62, 2**50 + 7, 777)])
def test_draws_bit_exact(orc, seed, step, base, n):
    need_gpu()
    import precision_label_chunk_b200 as elmo
    out = torch.empty(n, dtype=torch.int16, device="cuda")
    elmo.elmo_sr_draws(out, seed, step, base)
    got = out.cpu().numpy().view(np.uint16).astype(np.uint32)
    assert np.array_equal(got, orc.draw16(seed, step, base, n))


def test_sr_round_empty_and_errors():
    need_gpu()
    import precision_label_chunk_b200 as elmo
    x = torch.zeros(0, device="cuda")
    out = torch.zeros(0, dtype=torch.uint8, device="cuda")
    elmo.elmo_sr_round(x, out, "fp8", 0, 0)          # n = 0 is a no-op
    lib = elmo.load()
    assert lib.elmo_sr_round(None, None, 5, 0, 0, 0, 0, None) == 1      # null pointers: EINVAL
    assert lib.elmo_sr_round(None, None, -1, 0, 0, 0, 0, None) == 1     # n < 0: EINVAL
    xd = torch.zeros(4, device="cuda")
    assert lib.elmo_sr_round(xd.data_ptr(), out.data_ptr(), 4, 7, 0, 0, 0, None) == 1  # bad dtype
    # a head takes bf16, E4M3 or E5M2 weights; another format code is refused
    W = torch.zeros(128, 64, dtype=torch.uint8, device="cuda")
    h = ctypes.c_void_p()
    assert lib.elmo_init_head(ctypes.byref(h), W.data_ptr(), 128, 64, 9, 0, 0.0, 0, None) == 1        # EINVAL
