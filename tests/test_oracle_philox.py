"""Pins of the oracle's counter-based generator (Philox, Salmon et al. SC'11)
against independent library implementations and closed forms."""
import os
import shutil
import subprocess

import numpy as np
import pytest


def test_philox4x64_matches_numpy(orc):
    # numpy's Philox bit generator is the 4x64-10 member of the same family;
    # it increments its 256-bit counter and then emits the block of the new counter.
    rng = np.random.default_rng(7)
    for _ in range(20):
        key = rng.integers(0, 2**63, size=2, dtype=np.uint64) * np.uint64(2) + np.uint64(1)
        ctr = rng.integers(0, 2**63, size=4, dtype=np.uint64)
        ctr[0] = min(int(ctr[0]), 2**63 - 5)
        bg = np.random.Philox(key=key)
        st = bg.state
        st["state"]["counter"] = ctr.copy()
        bg.state = st
        got = bg.random_raw(4)
        nxt = ctr.copy()
        nxt[0] += np.uint64(1)
        assert np.array_equal(orc.philox4x64_10(nxt, key), got)


_CURAND_PROG = r"""
#define QUALIFIERS static inline __host__ __device__
#include <curand_philox4x32_x.h>
#include <cstdio>
int main() {
  unsigned a[6];
  while (scanf("%u %u %u %u %u %u", &a[0], &a[1], &a[2], &a[3], &a[4], &a[5]) == 6) {
    uint4 o = curand_Philox4x32_10(make_uint4(a[0], a[1], a[2], a[3]), make_uint2(a[4], a[5]));
    printf("%u %u %u %u\n", o.x, o.y, o.z, o.w);
  }
  return 0;
}
"""


@pytest.fixture(scope="module")
def curand_host(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("curand")
    src, exe = d / "p.cu", d / "p"
    src.write_text(_CURAND_PROG)
    subprocess.check_call([nvcc, "-Wno-deprecated-gpu-targets", "-o", str(exe), str(src)])
    return exe


def test_philox4x32_matches_curand_host(orc, curand_host):
    # cuRAND's Philox4x32-10, compiled for the host CPU, is an independent
    # implementation of the same published generator.
    rng = np.random.default_rng(11)
    rows = rng.integers(0, 2**32, size=(200, 6), dtype=np.uint64)
    rows[0] = 0
    rows[1] = 2**32 - 1
    inp = "\n".join(" ".join(str(int(v)) for v in r) for r in rows) + "\n"
    out = subprocess.run([str(curand_host)], input=inp, capture_output=True, text=True, check=True).stdout
    ref = np.array([[int(t) for t in line.split()] for line in out.strip().splitlines()], dtype=np.uint64)
    for r, e in zip(rows, ref):
        got = orc.philox4x32_10(r[:4].astype(np.uint32), r[4:].astype(np.uint32))
        assert np.array_equal(got.astype(np.uint64), e)


def test_draw16_layout_and_uniformity(orc):
    seed, step = 0x1234_5678_9ABC_DEF0, 17
    k = orc.draw16(seed, step, 0, 64)
    for blk in range(8):
        w = orc.philox4x32_10([blk, 0, step, 0], [seed & 0xFFFFFFFF, seed >> 32])
        halves = np.stack([w & 0xFFFF, w >> 16], axis=1).ravel()
        assert np.array_equal(k[8 * blk: 8 * blk + 8], halves)
    # chi-square over 256 bins of the top byte
    k = orc.draw16(3, 5, 10**9, 1 << 18)
    hist = np.bincount((k >> 8).astype(np.int64), minlength=256)
    exp = k.size / 256
    chi2 = float(((hist - exp) ** 2 / exp).sum())
    assert chi2 < 400  # 255 dof: mean 255, sd ~22.6
    # lag-1 serial correlation of the draws is ~0
    u = k.astype(np.float64) / 65536.0
    r = np.corrcoef(u[:-1], u[1:])[0, 1]
    assert abs(r) < 0.01
