"""CPU oracle for the ELMO classifier-head step (test infrastructure).

Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
leg of ``bench.py`` may import this package.  The product path never does:
it shares no code with the CUDA library.

The arithmetic lives in ``elmo_oracle.c`` (plain C, OpenMP over labels);
this module compiles it with gcc on first use and exposes numpy-level calls.
Every function cites the passage it follows in the C source.

Parity status: every function below is pinned by CPU tests
(tests/test_oracle_*.py) against library routines, closed forms, special
cases or float64 brute force.  Philox4x32-10 itself is pinned bit-exactly
against cuRAND's host implementation of the same generator (compiled from
the toolkit header and run, never copied), and the 4x64 member of the family
against numpy's Philox bit generator.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "elmo_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

BF16 = 0
FP8_E4M3 = 1
FP8_E4M3_GE5M2 = 2      # E4M3 weights and X, E5M2 gradient operand
FP8_E5M2 = 3            # E5M2 values; as a head: E5M2 weights with E4M3 X and gradient operand
_DT = {"bf16": BF16, "fp8": FP8_E4M3, "fp8_ge5m2": FP8_E4M3_GE5M2, "e5m2": FP8_E5M2, BF16: BF16,
       FP8_E4M3: FP8_E4M3, FP8_E4M3_GE5M2: FP8_E4M3_GE5M2, FP8_E5M2: FP8_E5M2}


def build(force: bool = False) -> str:
    """Compile the oracle (gcc, -O2, OpenMP, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=gnu11",
            "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            _lib = ctypes.CDLL(build())
            _declare(_lib)
    return _lib


def _declare(L):
    P = ctypes.c_void_p
    i64, i32, u64, f32 = ctypes.c_int64, ctypes.c_int32, ctypes.c_uint64, ctypes.c_float
    L.orc_philox4x32_10.argtypes = [P, P, P]
    L.orc_philox4x64_10.argtypes = [P, P, P]
    L.orc_draw16.argtypes = [u64, u64, u64]
    L.orc_draw16.restype = ctypes.c_uint32
    L.orc_draw16_array.argtypes = [u64, u64, u64, i64, P]
    L.orc_sr_bf16_array.argtypes = [P, P, i64, P]
    L.orc_sr_e4m3_array.argtypes = [P, P, i64, P]
    L.orc_sr_e5m2_array.argtypes = [P, P, i64, P]
    L.orc_rne_bf16_array.argtypes = [P, i64, P]
    L.orc_rne_e4m3_array.argtypes = [P, i64, P]
    L.orc_e4m3_value_array.argtypes = [P, i64, P]
    L.orc_rne_e5m2_array.argtypes = [P, i64, P]
    L.orc_e5m2_value_array.argtypes = [P, i64, P]
    L.orc_sr_round.argtypes = [P, P, i64, ctypes.c_int, u64, u64, u64]
    L.orc_fp8_x_scale.argtypes = [P, i64]
    L.orc_fp8_x_scale.restype = f32
    L.orc_train_step.argtypes = [P, P, i64, i32, ctypes.c_int, P, i32, P, P, f32, u64, u64,
                                 i64, i64, P, P, P, ctypes.c_int]
    L.orc_dx_rows.argtypes = [P, i64, i32, ctypes.c_int, P, i32, P, P, P, i32, P, P, P, ctypes.c_int]
    L.orc_topk.argtypes = [P, i64, i32, ctypes.c_int, P, i32, i32, P, i32, P, P, ctypes.c_int]
    L.orc_precision_at_k.argtypes = [P, i32, i32, P, P, P]
    L.orc_kahan_sgd.argtypes = [P, P, P, i64, f32]
    L.orc_scores.argtypes = [P, i64, i32, ctypes.c_int, P, i32, P, i32, i64, i64, P, ctypes.c_int]
    L.orc_score.argtypes = [P, ctypes.c_int, i64, P, i32, i32]
    L.orc_score.restype = f32


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


class OracleError(RuntimeError):
    pass


def _check(rc, what):
    if rc != 0:
        raise OracleError(f"{what} failed with code {rc}")


# ---------------------------------------------------------------- random bits
def philox4x32_10(ctr, key) -> np.ndarray:
    c, k, o = _c(ctr, np.uint32), _c(key, np.uint32), np.zeros(4, np.uint32)
    lib().orc_philox4x32_10(_p(c), _p(k), _p(o))
    return o


def philox4x64_10(ctr, key) -> np.ndarray:
    c, k, o = _c(ctr, np.uint64), _c(key, np.uint64), np.zeros(4, np.uint64)
    lib().orc_philox4x64_10(_p(c), _p(k), _p(o))
    return o


def draw16(seed: int, step: int, base: int, n: int) -> np.ndarray:
    """16-bit SR draws k of elements base .. base+n-1 (as uint32)."""
    o = np.zeros(n, np.uint32)
    lib().orc_draw16_array(seed, step, base, n, _p(o))
    return o


# ---------------------------------------------------------------- grids / SR
def sr_with_draws(v, k, dtype) -> np.ndarray:
    """SR of fp32 values v with explicit 16-bit draws k (same shape)."""
    v = _c(v, np.float32).ravel()
    k = _c(k, np.uint32).ravel()
    assert v.shape == k.shape
    if _DT[dtype] == BF16:
        o = np.zeros(v.shape, np.uint16)
        lib().orc_sr_bf16_array(_p(v), _p(k), v.size, _p(o))
    elif _DT[dtype] == FP8_E5M2:
        o = np.zeros(v.shape, np.uint8)
        lib().orc_sr_e5m2_array(_p(v), _p(k), v.size, _p(o))
    else:
        o = np.zeros(v.shape, np.uint8)
        lib().orc_sr_e4m3_array(_p(v), _p(k), v.size, _p(o))
    return o


def sr_round(x, dtype, seed: int, step: int, index_base: int = 0) -> np.ndarray:
    x = _c(x, np.float32)
    out = np.zeros(x.shape, np.uint16 if _DT[dtype] == BF16 else np.uint8)
    _check(lib().orc_sr_round(_p(x), _p(out), x.size, _DT[dtype], seed, step, index_base), "sr_round")
    return out


def rne_bf16(x) -> np.ndarray:
    x = _c(x, np.float32)
    o = np.zeros(x.shape, np.uint16)
    lib().orc_rne_bf16_array(_p(x), x.size, _p(o))
    return o


def rne_e4m3(x) -> np.ndarray:
    x = _c(x, np.float32)
    o = np.zeros(x.shape, np.uint8)
    lib().orc_rne_e4m3_array(_p(x), x.size, _p(o))
    return o


def e4m3_value(codes) -> np.ndarray:
    c = _c(codes, np.uint8)
    o = np.zeros(c.shape, np.float32)
    lib().orc_e4m3_value_array(_p(c), c.size, _p(o))
    return o


def rne_e5m2(x) -> np.ndarray:
    x = _c(x, np.float32)
    o = np.zeros(x.shape, np.uint8)
    lib().orc_rne_e5m2_array(_p(x), x.size, _p(o))
    return o


def e5m2_value(codes) -> np.ndarray:
    c = _c(codes, np.uint8)
    o = np.zeros(c.shape, np.float32)
    lib().orc_e5m2_value_array(_p(c), c.size, _p(o))
    return o


def bf16_value(bits) -> np.ndarray:
    return (_c(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def w_value(W, dtype) -> np.ndarray:
    dt = _DT[dtype]
    return bf16_value(W) if dt == BF16 else (e5m2_value(W) if dt == FP8_E5M2 else e4m3_value(W))


def fp8_x_scale(X) -> float:
    X = _c(X, np.uint16)
    return float(lib().orc_fp8_x_scale(_p(X), X.size))


# ---------------------------------------------------------------- the step
def train_step(W, X, rowptr, cols, lr, seed, step, dtype, l0=0, l1=None,
               want_dx=True, want_zg=False, nthreads=0, L=None):
    """One step over labels [l0, l1).  W: [L, d] uint16 (bf16) or uint8 (E4M3)
    codes; X: [B, d] bf16 bits.  Returns dict(W=[l1-l0, d] codes, dX=[B, d] fp32
    (contributions of those labels), Z/G=[l1-l0, B] fp32 when asked).
    L: total label count when W holds only the rows [0, l1) of a larger head."""
    dt = _DT[dtype]
    W = _c(W, np.uint16 if dt == BF16 else np.uint8)
    X = _c(X, np.uint16)
    Lw, d = W.shape
    L = Lw if L is None else L
    B = X.shape[0]
    assert X.shape[1] == d
    l1 = Lw if l1 is None else l1
    assert l1 <= Lw
    rowptr, cols = _c(rowptr, np.int32), _c(cols, np.int32)
    Wout = np.zeros((l1 - l0, d), W.dtype)
    dX = np.zeros((B, d), np.float32) if want_dx else None
    Z = np.zeros((l1 - l0, B), np.float32) if want_zg else None
    G = np.zeros((l1 - l0, B), np.float32) if want_zg else None
    _check(lib().orc_train_step(_p(W), _p(Wout), L, d, dt, _p(X), B, _p(rowptr), _p(cols),
                                lr, seed, step, l0, l1, _p(dX), _p(Z), _p(G), nthreads),
           "train_step")
    return {"W": Wout, "dX": dX, "Z": Z, "G": G}


def dx_rows(W, X, rowptr, cols, samples, dtype, nthreads=0, want_zg=False):
    """dX rows of the listed samples over all labels; with want_zg also their
    logits and gradient operand values ([len(samples), L] fp32 each):
    returns (dX rows, Z rows, G rows)."""
    dt = _DT[dtype]
    W = _c(W, np.uint16 if dt == BF16 else np.uint8)
    X = _c(X, np.uint16)
    L, d = W.shape
    samples = _c(samples, np.int32)
    out = np.zeros((samples.size, d), np.float32)
    Z = np.zeros((samples.size, L), np.float32) if want_zg else None
    G = np.zeros((samples.size, L), np.float32) if want_zg else None
    _check(lib().orc_dx_rows(_p(W), L, d, dt, _p(X), X.shape[0], _p(_c(rowptr, np.int32)),
                             _p(_c(cols, np.int32)), _p(samples), samples.size, _p(out), _p(Z), _p(G), nthreads),
           "dx_rows")
    return (out, Z, G) if want_zg else out


def topk(W, X, k, dtype, rows=None, nthreads=0):
    """Exact top-k (indices int32, scores fp32) for the listed rows of X."""
    dt = _DT[dtype]
    W = _c(W, np.uint16 if dt == BF16 else np.uint8)
    X = _c(X, np.uint16)
    L, d = W.shape
    B = X.shape[0]
    r = None if rows is None else _c(rows, np.int32)
    n = B if r is None else r.size
    idx = np.zeros((n, k), np.int32)
    sc = np.zeros((n, k), np.float32)
    _check(lib().orc_topk(_p(W), L, d, dt, _p(X), B, k, _p(r), n, _p(idx), _p(sc), nthreads), "topk")
    return idx, sc


def precision_at_k(idx, rowptr, cols):
    """P@1 .. P@k (float64 [k]) of predictions idx [B, k] against CSR positives."""
    idx = _c(idx, np.int32)
    B, k = idx.shape
    p = np.zeros(k, np.float64)
    _check(lib().orc_precision_at_k(_p(idx), B, k, _p(_c(rowptr, np.int32)), _p(_c(cols, np.int32)), _p(p)),
           "precision_at_k")
    return p


def kahan_sgd(p, c, g, lr):
    """One Kahan-compensated SGD step of bf16 parameters p with bf16
    compensation c and bf16 gradient g (uint16 bit patterns, same shape).
    Returns the new (p, c)."""
    p = _c(p, np.uint16).copy()
    c = _c(c, np.uint16).copy()
    g = _c(g, np.uint16)
    assert p.shape == c.shape == g.shape
    lib().orc_kahan_sgd(_p(p), _p(c), _p(g), p.size, float(lr))
    return p, c


def scores(W, X, rows, l0, l1, dtype, nthreads=0) -> np.ndarray:
    """Exact top-k scores (the fp32 fma chain) of the listed rows of X against
    labels [l0, l1): fp32 [len(rows), l1 - l0]."""
    dt = _DT[dtype]
    W = _c(W, np.uint16 if dt == BF16 else np.uint8)
    X = _c(X, np.uint16)
    L, d = W.shape
    rows = _c(rows, np.int32)
    out = np.zeros((rows.size, l1 - l0), np.float32)
    _check(lib().orc_scores(_p(W), L, d, dt, _p(X), X.shape[0], _p(rows), rows.size, l0, l1, _p(out), nthreads),
           "scores")
    return out


def score(W, X, l, b, dtype) -> float:
    dt = _DT[dtype]
    W = _c(W, np.uint16 if dt == BF16 else np.uint8)
    X = _c(X, np.uint16)
    return float(lib().orc_score(_p(W), dt, l, _p(X), b, W.shape[1]))
