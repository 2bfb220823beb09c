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
