"""Helpers of the GPU parity tests: move seeded inputs to the device and run
the library through its C ABI (via the binding)."""
import numpy as np
import pytest
import torch


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def to_dev_u16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def to_dev_u8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def to_dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def w_to_dev(W, dtype):
    return to_dev_u16(W) if dtype == "bf16" else to_dev_u8(W)


def w_to_host(Wd, dtype):
    a = Wd.cpu().numpy()
    return a.view(np.uint16) if dtype == "bf16" else a.view(np.uint8)


def run_step(elmo, W, X, rowptr, cols, lr, chunk, seed, step, dtype, head=None):
    """One library step on device copies; returns (new W codes, dX, head, Wd)."""
    Wd = w_to_dev(W, dtype)
    h = elmo.elmo_init_head(Wd, dtype)
    Xd = to_dev_u16(X)
    dX = torch.empty(X.shape[0], X.shape[1], dtype=torch.float32, device="cuda")
    elmo.elmo_train_step_chunked(h, Xd, to_dev_i32(rowptr), to_dev_i32(cols), lr, chunk, seed, step, dX)
    elmo.elmo_sync_status(h)
    out = w_to_host(Wd, dtype), dX.cpu().numpy()
    h.close()
    return out


def run_step_with_operands(elmo, W, X, rowptr, cols, lr, chunk, seed, step, dtype, span=1 << 16):
    """The logits and gradient operands of every label (forward_chunk, over
    ranges of `span` labels; W untouched), then one step on the same head.
    Returns (new W codes, dX, Z [L, B], G [L, B])."""
    Wd = w_to_dev(W, "bf16" if dtype == "bf16" else "fp8")     # one byte per code for every 8-bit grid
    h = elmo.elmo_init_head(Wd, dtype)
    Xd, rp, cl = to_dev_u16(X), to_dev_i32(rowptr), to_dev_i32(cols)
    L, B = W.shape[0], X.shape[0]
    Z = np.empty((L, B), np.float32)
    G = np.empty((L, B), np.float32)
    for a in range(0, L, span):
        e = min(L, a + span)
        Zd = torch.empty(e - a, B, device="cuda")
        Gd = torch.empty(e - a, B, device="cuda")
        elmo.elmo_forward_chunk(h, Xd, rp, cl, a, e, Zd, Gd)
        Z[a:e], G[a:e] = Zd.cpu().numpy(), Gd.cpu().numpy()
    dX = torch.empty(B, X.shape[1], dtype=torch.float32, device="cuda")
    elmo.elmo_train_step_chunked(h, Xd, rp, cl, lr, chunk, seed, step, dX)
    elmo.elmo_sync_status(h)
    out = w_to_host(Wd, "bf16" if dtype == "bf16" else "fp8"), dX.cpu().numpy(), Z, G
    h.close()
    return out
