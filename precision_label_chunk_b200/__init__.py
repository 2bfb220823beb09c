"""Python binding of libelmo, the B200 (sm_100a) ELMO classifier-head library.

Argument marshalling only: every call below forwards device pointers of
torch tensors and the current CUDA stream to the C ABI declared in
include/elmo.h, whose kernels do all of the work.  There is no fallback: if
libelmo.so is missing or cannot be loaded, importing the library functions
raises.

The names match the C entry points:
  elmo_init_head, elmo_init_head_shard, elmo_head_destroy,
  elmo_train_step_chunked, elmo_train_step_noalloc, elmo_forward_chunk,
  elmo_topk_predict, elmo_topk_merge, elmo_sr_round, elmo_sr_draws,
  elmo_precision_at_k, elmo_kahan_sgd, elmo_round_bf16,
  elmo_check_bounded_wait, elmo_sync_status,
  elmo_head_workspace_bytes and the tracing calls.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = [
    "ElmoError", "Head", "BF16", "FP8_E4M3", "FP8_E4M3_GE5M2", "FP8_E5M2", "MAX_BATCH", "MAX_NNZ", "MAX_TOPK", "MAX_PREDICT_BATCH",
    "library_path", "load", "elmo_init_head", "elmo_head_destroy", "elmo_train_step_chunked",
    "elmo_forward_chunk", "elmo_topk_predict", "elmo_topk_uncertified_rows", "elmo_topk_screen_scores",
    "elmo_sr_round", "elmo_sr_draws",
    "elmo_sync_status", "elmo_head_workspace_bytes", "elmo_profile_enable", "elmo_profile_reset",
    "elmo_profile_read", "elmo_launch_count", "KERNEL_CLASSES", "elmo_train_step_noalloc",
    "elmo_check_bounded_wait", "WAIT_CHECK_SITE", "elmo_precision_at_k", "elmo_init_head_shard",
    "elmo_topk_merge", "MAX_SHARDS", "MAX_TOTAL_LABELS", "elmo_kahan_sgd", "elmo_round_bf16", "elmo_last_error",
]

BF16 = 0
FP8_E4M3 = 1
FP8_E4M3_GE5M2 = 2    # E4M3 weights, E5M2 gradient operand in the training step
FP8_E5M2 = 3          # E5M2 values: an SR output grid, and heads with E5M2 weights (E4M3 X and G)
WAIT_CHECK_SITE = 99
MAX_BATCH = 256
MAX_NNZ = 32768
MAX_TOPK = 64
MAX_PREDICT_BATCH = 4096
MAX_TOTAL_LABELS = 2**31 - 1
MAX_SHARDS = 64

STATUS_NAMES = {0: "ELMO_OK", 1: "ELMO_EINVAL", 2: "ELMO_ENOMEM", 3: "ELMO_ECUDA", 4: "ELMO_ETIMEOUT",
                5: "ELMO_EUNSUPPORTED", 6: "ELMO_EDATA"}

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None
_lock = threading.Lock()


class ElmoError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def library_path() -> str:
    return os.path.join(_HERE, "libelmo.so")


def load():
    """Load libelmo.so (built in-tree by __graft_entry__.build())."""
    global _lib
    with _lock:
        if _lib is None:
            path = library_path()
            if not os.path.exists(path):
                raise ImportError(f"libelmo.so not found at {path}; build it with "
                                  "`python -m precision_label_chunk_b200._build`")
            lib = ctypes.CDLL(path)
            _declare(lib)
            _lib = lib
    return _lib


def _declare(L):
    P, i32, i64, u64, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_float
    st = ctypes.c_int
    L.elmo_last_error.restype = ctypes.c_char_p
    L.elmo_init_head.argtypes = [ctypes.POINTER(P), P, i64, i32, ctypes.c_int, ctypes.c_int, f32, u64, P]
    L.elmo_init_head_shard.argtypes = [ctypes.POINTER(P), P, i64, i32, ctypes.c_int, i64, i64, ctypes.c_int, f32,
                                       u64, P]
    L.elmo_topk_merge.argtypes = [P, P, i32, i32, i32, P, P, P]
    L.elmo_kahan_sgd.argtypes = [P, P, P, i64, f32, P]
    L.elmo_round_bf16.argtypes = [P, P, i64, P]
    L.elmo_head_destroy.argtypes = [P]
    L.elmo_train_step_chunked.argtypes = [P, P, i32, P, P, i32, f32, i64, u64, u64, P, P]
    L.elmo_forward_chunk.argtypes = [P, P, i32, P, P, i32, i64, i64, P, P, P]
    L.elmo_topk_predict.argtypes = [P, P, i32, i32, i64, P, P, P]
    L.elmo_topk_uncertified_rows.argtypes = [P, i32, i32, ctypes.POINTER(i32), P]
    L.elmo_topk_screen_scores.argtypes = [P, P, i32, i64, i64, P, P, P]
    L.elmo_sr_round.argtypes = [P, P, i64, ctypes.c_int, u64, u64, u64, P]
    L.elmo_sr_draws.argtypes = [P, i64, u64, u64, u64, P]
    L.elmo_sync_status.argtypes = [P, P]
    L.elmo_head_workspace_bytes.argtypes = [P, ctypes.POINTER(ctypes.c_size_t)]
    L.elmo_train_step_noalloc.argtypes = [P, i64, i32, ctypes.c_int, P, i32, P, P, i32, f32, i64, u64, u64, P, P, P]
    L.elmo_train_step_noalloc.restype = st
    L.elmo_profile_enable.argtypes = [P, ctypes.c_int]
    L.elmo_profile_reset.argtypes = [P]
    L.elmo_profile_read.argtypes = [P, ctypes.c_int, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(i64)]
    L.elmo_launch_count.argtypes = [P, ctypes.POINTER(i64)]
    L.elmo_check_bounded_wait.argtypes = [i64, P, P]
    L.elmo_precision_at_k.argtypes = [P, i32, i32, P, P, i32, P, P]
    for name in ("elmo_profile_enable", "elmo_profile_reset", "elmo_profile_read", "elmo_launch_count","elmo_init_head", "elmo_head_destroy", "elmo_train_step_chunked", "elmo_forward_chunk",
                 "elmo_topk_predict", "elmo_sr_round", "elmo_sr_draws", "elmo_sync_status",
                 "elmo_head_workspace_bytes", "elmo_topk_uncertified_rows", "elmo_topk_screen_scores"):
        getattr(L, name).restype = st


def elmo_last_error() -> str:
    """The message of this thread's last failed call ("" after a success)."""
    return load().elmo_last_error().decode(errors="replace")


def _check(rc: int):
    if rc != 0:
        raise ElmoError(rc, elmo_last_error())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _dt(dtype) -> int:
    if dtype in (BF16, "bf16", torch.bfloat16):
        return BF16
    if dtype in (FP8_E4M3, "fp8", "e4m3", torch.float8_e4m3fn):
        return FP8_E4M3
    if dtype in (FP8_E4M3_GE5M2, "fp8_ge5m2"):
        return FP8_E4M3_GE5M2
    if dtype in (FP8_E5M2, "e5m2", torch.float8_e5m2):
        return FP8_E5M2
    raise ValueError(f"unknown dtype {dtype!r}")


class Head:
    """A borrowed weight matrix W [L, d] plus the library's workspace; W holds
    the label rows [label_base, label_base + L) of a head of labels_total."""

    def __init__(self, handle: ctypes.c_void_p, W: torch.Tensor, dtype: int, label_base: int = 0,
                 labels_total: int | None = None):
        self.handle = handle
        self.W = W
        self.dtype = dtype
        self.L, self.d = W.shape
        self.label_base = label_base
        self.labels_total = self.L if labels_total is None else labels_total

    def close(self):
        if self.handle:
            _check(load().elmo_head_destroy(self.handle))
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def elmo_init_head(W: torch.Tensor, dtype=None, fill: bool = False, init_std: float = 0.02, seed: int = 0,
                   stream=None) -> Head:
    """A head over W: [L, d] CUDA tensor of bf16 values ("bf16") or E4M3 codes
    ("fp8"; "fp8_ge5m2" for the step with an E5M2 gradient operand), borrowed
    and updated in place by the training steps.  fill=True overwrites W with
    SR(init_std * N(0, 1)) drawn from Philox keyed by seed."""
    return elmo_init_head_shard(W, 0, W.shape[0], dtype, fill, init_std, seed, stream)


def elmo_init_head_shard(W: torch.Tensor, label_base: int, labels_total: int, dtype=None, fill: bool = False,
                         init_std: float = 0.02, seed: int = 0, stream=None) -> Head:
    """W: this device's label rows [label_base, label_base + L) of a head of
    labels_total labels split by labels over several devices."""
    if dtype is None:
        dtype = BF16 if W.dtype in (torch.bfloat16, torch.int16) else FP8_E4M3
    dt = _dt(dtype)
    if W.dim() != 2:
        raise ValueError("W must be 2-D [L, d]")
    if W.element_size() != (2 if dt == BF16 else 1):
        raise ValueError("W element size does not match dtype")
    h = ctypes.c_void_p()
    _check(load().elmo_init_head_shard(ctypes.byref(h), _ptr(W), W.shape[0], W.shape[1], dt, int(label_base),
                                       int(labels_total), int(bool(fill)), float(init_std), int(seed) & (2**64 - 1),
                                       _stream(stream)))
    return Head(h, W, dt, int(label_base), int(labels_total))


def elmo_head_destroy(head: Head):
    head.close()


def elmo_train_step_chunked(head: Head, X: torch.Tensor, rowptr: torch.Tensor, cols: torch.Tensor, lr: float,
                            chunk: int, seed: int, step: int, dX: torch.Tensor, stream=None):
    """One fused SGD step of the head: X bf16 [B, d], CSR positives rowptr
    [B + 1] / cols [nnz] (int32, label ids of the whole head), chunk labels per
    chunk; W is updated in place with stochastic rounding of stream (seed,
    step) and dX (fp32 [B, d]) receives the input gradient."""
    B = X.shape[0]
    nnz = cols.numel()
    _check(load().elmo_train_step_chunked(head.handle, _ptr(X), B, _ptr(rowptr), _ptr(cols) if nnz else None,
                                          nnz, float(lr), int(chunk), int(seed) & (2**64 - 1),
                                          int(step) & (2**64 - 1), _ptr(dX), _stream(stream)))


def elmo_train_step_noalloc(W: torch.Tensor, dtype, X: torch.Tensor, rowptr: torch.Tensor, cols: torch.Tensor,
                            lr: float, chunk: int, seed: int, step: int, dX: torch.Tensor, status: torch.Tensor,
                            stream=None):
    """The training step without a head and without any device allocation, for
    callers that must not allocate (stream capture, fixed memory budgets).
    W: [L, d] weights (updated in place); status: int32 [2] device tensor that
    receives ELMO_EDATA for malformed labels.  See include/elmo.h."""
    nnz = cols.numel()
    _check(load().elmo_train_step_noalloc(_ptr(W), W.shape[0], W.shape[1], _dt(dtype), _ptr(X), X.shape[0],
                                          _ptr(rowptr), _ptr(cols) if nnz else None, nnz, float(lr), int(chunk),
                                          int(seed) & (2**64 - 1), int(step) & (2**64 - 1), _ptr(dX), _ptr(status),
                                          _stream(stream)))


def elmo_forward_chunk(head: Head, X: torch.Tensor, rowptr: torch.Tensor, cols: torch.Tensor, l0: int, l1: int,
                       Z: torch.Tensor | None = None, G: torch.Tensor | None = None, stream=None):
    """Inspection: logits Z and rounded gradient operand values G (fp32
    [l1 - l0, B]) of rows [l0, l1) as the step forms them; W is not touched."""
    nnz = cols.numel()
    _check(load().elmo_forward_chunk(head.handle, _ptr(X), X.shape[0], _ptr(rowptr), _ptr(cols) if nnz else None,
                                     nnz, int(l0), int(l1), _ptr(Z), _ptr(G), _stream(stream)))


def elmo_topk_predict(head: Head, X: torch.Tensor, k: int, chunk: int, idx: torch.Tensor, score: torch.Tensor,
                      stream=None):
    """Top-k labels per row of X (bf16 [B, d]): idx int32 [B, k] (label ids of
    the whole head, best first) and score fp32 [B, k], the exact fp32 chain."""
    _check(load().elmo_topk_predict(head.handle, _ptr(X), X.shape[0], int(k), int(chunk), _ptr(idx), _ptr(score),
                                    _stream(stream)))


def elmo_topk_uncertified_rows(head: Head, B: int, k: int, stream=None) -> int:
    """Rows of the last elmo_topk_predict(B, k) on this head that the screening
    certificate sent to the exact path."""
    n = ctypes.c_int32()
    _check(load().elmo_topk_uncertified_rows(head.handle, int(B), int(k), ctypes.byref(n), _stream(stream)))
    return int(n.value)


def elmo_topk_screen_scores(head: Head, X: torch.Tensor, l0: int, l1: int, S: torch.Tensor, bound: torch.Tensor,
                            stream=None):
    """Inspection: the tensor-core screening scores S (fp32 [B, l1 - l0]) of
    labels [l0, l1) and each row's certificate bound (fp32 [B])."""
    _check(load().elmo_topk_screen_scores(head.handle, _ptr(X), X.shape[0], int(l0), int(l1), _ptr(S), _ptr(bound),
                                          _stream(stream)))


def elmo_topk_merge(idx: torch.Tensor, score: torch.Tensor, idx_out: torch.Tensor, score_out: torch.Tensor,
                    stream=None):
    """Top-k of a head split over P devices: idx/score [P, B, k] (each device's
    list, best first) -> idx_out/score_out [B, k]."""
    P, B, k = idx.shape
    _check(load().elmo_topk_merge(_ptr(idx), _ptr(score), P, B, k, _ptr(idx_out), _ptr(score_out), _stream(stream)))


def elmo_kahan_sgd(p: torch.Tensor, c: torch.Tensor, g: torch.Tensor, lr: float, stream=None):
    """One Kahan-compensated SGD step: bf16 parameters p and compensation c
    (updated in place) with bf16 gradient g, all of the same size."""
    if not (p.numel() == c.numel() == g.numel()) or any(t.element_size() != 2 for t in (p, c, g)):
        raise ValueError("p, c and g must be bf16 tensors of the same size")
    _check(load().elmo_kahan_sgd(_ptr(p), _ptr(c), _ptr(g), p.numel(), float(lr), _stream(stream)))


def elmo_round_bf16(inp: torch.Tensor, out: torch.Tensor, stream=None):
    """out = bf16(inp), round to nearest-even (fp32 dX handed to a bf16 encoder)."""
    if inp.numel() != out.numel() or out.element_size() != 2:
        raise ValueError("out must be a 2-byte tensor of inp's size")
    _check(load().elmo_round_bf16(_ptr(inp), _ptr(out), inp.numel(), _stream(stream)))


def elmo_sr_round(inp: torch.Tensor, out: torch.Tensor, dtype, seed: int, step: int, index_base: int = 0,
                  stream=None):
    """out = SR(inp) onto the "bf16", "fp8" (E4M3) or "e5m2" grid with the draws
    of elements index_base .. of stream (seed, step)."""
    _check(load().elmo_sr_round(_ptr(inp), _ptr(out), inp.numel(), _dt(dtype), int(seed) & (2**64 - 1),
                                int(step) & (2**64 - 1), int(index_base) & (2**64 - 1), _stream(stream)))


def elmo_sr_draws(out: torch.Tensor, seed: int, step: int, index_base: int = 0, stream=None):
    """The 16-bit draws (uint16 in a 2-byte tensor) that SR uses for elements index_base .."""
    _check(load().elmo_sr_draws(_ptr(out), out.numel(), int(seed) & (2**64 - 1), int(step) & (2**64 - 1),
                                int(index_base) & (2**64 - 1), _stream(stream)))


def elmo_precision_at_k(idx: torch.Tensor, rowptr: torch.Tensor, cols: torch.Tensor, p: torch.Tensor, stream=None):
    """P@1 .. P@k (fp32 [k], device) of predictions idx (int32 [B, k], device)
    against the CSR positives rowptr/cols (int32, device)."""
    B, k = idx.shape
    _check(load().elmo_precision_at_k(_ptr(idx), B, k, _ptr(rowptr), _ptr(cols), cols.numel(), _ptr(p),
                                      _stream(stream)))


def elmo_check_bounded_wait(limit_cycles: int, status: torch.Tensor, stream=None):
    """Runs the kernels' bounded mbarrier wait on a barrier nothing arrives on;
    after synchronising, status (int32 [2], device) holds ELMO_ETIMEOUT and
    WAIT_CHECK_SITE."""
    _check(load().elmo_check_bounded_wait(int(limit_cycles), _ptr(status), _stream(stream)))


def elmo_sync_status(head: Head, stream=None):
    """Synchronise and raise ElmoError if a kernel recorded ELMO_EDATA or ELMO_ETIMEOUT (then cleared)."""
    _check(load().elmo_sync_status(head.handle, _stream(stream)))


KERNEL_CLASSES = {"prep": 0, "logits_grad": 1, "input_grad": 2, "update": 3, "topk_score": 4, "topk_merge": 5,
                  "other": 6, "step": 7}


def elmo_profile_enable(head: Head, enable: bool = True):
    _check(load().elmo_profile_enable(head.handle, int(bool(enable))))


def elmo_profile_reset(head: Head):
    _check(load().elmo_profile_reset(head.handle))


def elmo_profile_read(head: Head, kernel_class) -> tuple[float, int]:
    """(summed device milliseconds, launches) of one kernel class since the last reset."""
    cls = KERNEL_CLASSES[kernel_class] if isinstance(kernel_class, str) else int(kernel_class)
    ms, n = ctypes.c_double(), ctypes.c_int64()
    _check(load().elmo_profile_read(head.handle, cls, ctypes.byref(ms), ctypes.byref(n)))
    return float(ms.value), int(n.value)


def elmo_launch_count(head: Head) -> int:
    n = ctypes.c_int64()
    _check(load().elmo_launch_count(head.handle, ctypes.byref(n)))
    return int(n.value)


def elmo_head_workspace_bytes(head: Head) -> int:
    n = ctypes.c_size_t()
    _check(load().elmo_head_workspace_bytes(head.handle, ctypes.byref(n)))
    return int(n.value)
