"""Seeded synthetic workloads shaped like the ELMO classifier-head benchmarks.

This module only draws random inputs.  It holds none of the method's
arithmetic (no logits, no gradients, no rounding rules of the method), so the
CUDA path and the CPU oracle can both consume exactly the same bytes.

Workload shapes follow the dataset sizes named on the ELMO pages
("ELMO: Efficiency via Low-precision and Peak Memory Optimization in Large
Output Spaces", Key results: Wiki-500K, Amazon-3M, LF-Paper2Keywords-8.6M).
The datasets themselves are not available; nothing here reproduces any of
their records.  Labels are synthetic: every sample gets 1 + Poisson(lam)
distinct positive labels drawn from a truncated Zipf(s) law over label ranks
1..L (inverse CDF on the finite weights), mapped through a fixed seeded
permutation of [0, L) so that the frequent labels are spread over all chunks.

Values:
  X ~ N(0, 1) / sqrt(d)   (the tiny workload uses N(0, 1)), rounded to bf16 (RNE)
  W ~ N(0, 0.02^2) as fp32; bf16 workloads round it to bf16 (RNE); fp8
      workloads hand the fp32 values to the stochastic-rounding routine of
      whichever side (GPU or oracle) consumes them.
"""
from __future__ import annotations

import dataclasses
import functools

import numpy as np
import torch

__all__ = [
    "Workload", "WORKLOADS", "workload", "make_X", "make_W_f32", "make_W_bf16",
    "make_labels", "bf16_bits", "bf16_value", "labels_dense",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int            # seed namespace of the workload
    B: int                # samples per step
    d: int                # embedding width
    L: int                # number of labels
    dtype: str            # "bf16" or "fp8" (storage type of W); "fp8_ge5m2": E4M3 W, E5M2 gradient operand;
                          # "e5m2": E5M2 W (E4M3 X and gradient operand)
    lam: float            # positives per sample: 1 + Poisson(lam)
    zipf_s: float         # Zipf exponent of the label law
    lr: float
    chunk: int            # label chunk the caller passes to the step
    steps: int            # consecutive steps of the workload
    x_scale_by_sqrt_d: bool = True
    topk: int = 0         # >0: a prediction workload (top-k), no training


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny", 0, B=32, d=64, L=4096, dtype="bf16", lam=5, zipf_s=1.1,
                 lr=0.05, chunk=1024, steps=1, x_scale_by_sqrt_d=False),
        Workload("text500k_bf16", 1, B=256, d=768, L=500_000, dtype="bf16", lam=4,
                 zipf_s=1.1, lr=0.05, chunk=65_536, steps=20),
        Workload("product3m_fp8", 2, B=256, d=768, L=3_000_000, dtype="fp8", lam=35,
                 zipf_s=1.0, lr=0.1, chunk=131_072, steps=20),
        Workload("keyword8m6_bf16", 3, B=128, d=768, L=8_600_000, dtype="bf16", lam=10,
                 zipf_s=1.2, lr=0.05, chunk=262_144, steps=10),
        Workload("topk5_3m_fp8", 4, B=1024, d=768, L=3_000_000, dtype="fp8", lam=0,
                 zipf_s=1.0, lr=0.0, chunk=131_072, steps=1, topk=5),
        # the 3M-label head with an E5M2 gradient operand (same inputs as product3m_fp8)
        Workload("product3m_fp8_ge5m2", 2, B=256, d=768, L=3_000_000, dtype="fp8_ge5m2", lam=35,
                 zipf_s=1.0, lr=0.1, chunk=131_072, steps=20),
        # the 3M-label head with E5M2 weights (same inputs as product3m_fp8)
        Workload("product3m_e5m2", 2, B=256, d=768, L=3_000_000, dtype="e5m2", lam=35,
                 zipf_s=1.0, lr=0.1, chunk=131_072, steps=20),
    ]
}


def workload(name: str, **overrides) -> Workload:
    """A named workload, optionally with some fields replaced (smaller L, B ...)."""
    return dataclasses.replace(WORKLOADS[name], **overrides)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round-to-nearest-even via torch."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_value(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> fp32 values."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def make_X(w: Workload, step: int) -> np.ndarray:
    """X [B, d] as bf16 bit patterns (uint16)."""
    rng = np.random.default_rng([1000 + w.index, step, 1])
    x = rng.standard_normal((w.B, w.d), dtype=np.float32)
    if w.x_scale_by_sqrt_d:
        x /= np.float32(np.sqrt(w.d))
    return bf16_bits(x)


def make_W_f32(w: Workload, std: float = 0.02, rows: int | None = None) -> np.ndarray:
    """W [L, d] ~ N(0, std^2) as fp32 (before any rounding to the storage grid).
    rows: only the first `rows` label rows (the same values as the full draw)."""
    rng = np.random.default_rng([2000 + w.index])
    out = rng.standard_normal((w.L if rows is None else min(rows, w.L), w.d), dtype=np.float32)
    out *= np.float32(std)
    return out


def make_W_bf16(w: Workload, std: float = 0.02) -> np.ndarray:
    """W [L, d] ~ N(0, std^2) rounded (RNE) to bf16, as uint16 bit patterns."""
    return bf16_bits(make_W_f32(w, std))


@functools.lru_cache(maxsize=8)
def _zipf_cdf(L: int, s: float) -> np.ndarray:
    ranks = np.arange(1, L + 1, dtype=np.float64)
    wts = ranks ** (-float(s))
    cdf = np.cumsum(wts)
    cdf /= cdf[-1]
    return cdf


@functools.lru_cache(maxsize=8)
def _label_perm(L: int, index: int) -> np.ndarray:
    return np.random.default_rng([3000 + index]).permutation(L).astype(np.int32)


def make_labels(w: Workload, step: int, lam: float | None = None):
    """Sparse positives as CSR: (rowptr int32 [B+1], cols int32 [nnz]).

    Every sample has 1 + Poisson(lam) distinct labels (capped at L), drawn
    from the truncated Zipf(s) law and permuted.  Columns of a row are in
    draw order (not sorted), which the consumers must accept.
    """
    lam = w.lam if lam is None else lam
    rng = np.random.default_rng([1000 + w.index, step, 2])
    cdf = _zipf_cdf(w.L, w.zipf_s)
    perm = _label_perm(w.L, w.index)
    counts = np.minimum(1 + rng.poisson(lam, size=w.B), w.L)
    rows = []
    for c in counts:
        got: list[int] = []
        seen: set[int] = set()
        while len(got) < c:
            u = rng.random(int(2 * (c - len(got)) + 4))
            ranks = np.searchsorted(cdf, u, side="right")
            ranks = np.minimum(ranks, w.L - 1)
            for r in ranks:
                lab = int(perm[r])
                if lab not in seen:
                    seen.add(lab)
                    got.append(lab)
                    if len(got) == c:
                        break
        rows.append(np.asarray(got, dtype=np.int32))
    rowptr = np.zeros(w.B + 1, dtype=np.int32)
    rowptr[1:] = np.cumsum([len(r) for r in rows])
    cols = np.concatenate(rows).astype(np.int32) if rows else np.zeros(0, np.int32)
    return rowptr, cols


def labels_dense(rowptr: np.ndarray, cols: np.ndarray, L: int, l0: int = 0, l1: int | None = None):
    """Dense 0/1 matrix Y[b, l - l0] for labels in [l0, l1) (test helper)."""
    l1 = L if l1 is None else l1
    B = len(rowptr) - 1
    Y = np.zeros((B, l1 - l0), dtype=np.float32)
    for b in range(B):
        for c in cols[rowptr[b]:rowptr[b + 1]]:
            if l0 <= c < l1:
                Y[b, c - l0] = 1.0
    return Y
