"""Memory-safety checks without a sanitizer: guard bands around every buffer a
call writes, and the library's answer when the device runs out of memory.

Each caller buffer (W, dX, top-k outputs, SR outputs, inspection outputs) is
placed inside a larger allocation filled with a byte pattern; after ragged
steps, top-k calls and SR rounding, the bytes before and after each buffer
must still hold the pattern.  The out-of-memory case fills the device with a
single torch allocation first, so that the library's own cudaMalloc fails and
must come back as ELMO_ENOMEM with the device still usable."""
import numpy as np
import pytest
import torch

from synthetic import make_labels, make_W_f32, make_X, workload
from tests.gpu_common import need_gpu, to_dev_i32, to_dev_u16

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes on each side (keeps every buffer 16-byte aligned)
PATTERN = 0xA5


class Guarded:
    """A device buffer of `nbytes` with guard bands on both sides."""

    def __init__(self, nbytes):
        self.n = nbytes
        self.raw = torch.full((nbytes + 2 * GUARD,), PATTERN, dtype=torch.uint8, device="cuda")

    def view(self, dtype, shape):
        return self.raw[GUARD:GUARD + self.n].view(dtype).view(*shape)

    def intact(self):
        torch.cuda.synchronize()
        head = self.raw[:GUARD].cpu().numpy()
        tail = self.raw[GUARD + self.n:].cpu().numpy()
        return bool(np.all(head == PATTERN) and np.all(tail == PATTERN))


@pytest.mark.parametrize("dtype,L,d,B", [("fp8", 1000, 768, 256), ("bf16", 777, 128, 100), ("fp8", 300, 4096, 7),
                                         ("bf16", 2000, 768, 256)])
def test_guard_bands_around_step_and_topk(orc, dtype, L, d, B):
    """Ragged label counts (not a multiple of 128), a padded batch and each
    kernel family of the step (persistent, resident-X, streamed) and of top-k."""
    need_gpu()
    import precision_label_chunk_b200 as elmo
    w = workload("tiny", dtype=dtype, L=L, d=d, B=B)
    esz = 1 if dtype == "fp8" else 2
    W0 = make_W_f32(w)
    codes = orc.sr_round(W0, dtype, 0, 2**64 - 1)
    gW = Guarded(L * d * esz)
    Wd = gW.view(torch.uint8 if dtype == "fp8" else torch.int16, (L, d))
    Wd.copy_(torch.from_numpy(codes.view(np.uint8 if dtype == "fp8" else np.int16)).cuda())
    gdx = Guarded(B * d * 4)
    dX = gdx.view(torch.float32, (B, d))
    h = elmo.elmo_init_head(Wd, dtype)
    X = to_dev_u16(make_X(w, 0))
    rowptr, cols = make_labels(w, 0)
    for step in range(2):
        elmo.elmo_train_step_chunked(h, X, to_dev_i32(rowptr), to_dev_i32(cols), w.lr, 512, 1, step, dX)
    gz, gg = Guarded(L * B * 4), Guarded(L * B * 4)
    elmo.elmo_forward_chunk(h, X, to_dev_i32(rowptr), to_dev_i32(cols), 0, L, gz.view(torch.float32, (L, B)),
                            gg.view(torch.float32, (L, B)))
    k = 5
    gi, gs = Guarded(B * k * 4), Guarded(B * k * 4)
    elmo.elmo_topk_predict(h, X, k, 512, gi.view(torch.int32, (B, k)), gs.view(torch.float32, (B, k)))
    elmo.elmo_sync_status(h)
    for name, g in [("W", gW), ("dX", gdx), ("Z", gz), ("G", gg), ("top-k idx", gi), ("top-k score", gs)]:
        assert g.intact(), f"a kernel wrote outside {name}"
    h.close()


def test_guard_bands_around_sr_round():
    need_gpu()
    import precision_label_chunk_b200 as elmo
    n = 1000003                                           # a ragged tail after the 16-value blocks
    x = torch.randn(n, device="cuda") * 0.02
    for dt, esz in (("fp8", 1), ("bf16", 2), ("e5m2", 1)):
        g = Guarded(n * esz)
        out = g.view(torch.uint8 if esz == 1 else torch.int16, (n,))
        elmo.elmo_sr_round(x, out, dt, 3, 4, 5)
        assert g.intact(), f"SR onto {dt} wrote outside its output"


def test_out_of_device_memory_is_reported():
    """With the device full, the step's first call (which allocates its
    transient gradient-operand buffer, 8 MB or more) returns ELMO_ENOMEM
    instead of running; with memory back the same head steps normally."""
    need_gpu()
    import precision_label_chunk_b200 as elmo
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    W = torch.zeros(4096, 768, dtype=torch.uint8, device="cuda")
    h = elmo.elmo_init_head(W, "fp8")
    X = torch.zeros(8, 768, dtype=torch.bfloat16, device="cuda")
    dX = torch.empty(8, 768, device="cuda")
    rowptr = torch.zeros(9, dtype=torch.int32, device="cuda")
    cols = torch.zeros(0, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    free, _ = torch.cuda.mem_get_info()
    hog = torch.empty(max(0, free - (4 << 20)), dtype=torch.uint8, device="cuda")   # all but about 4 MiB
    try:
        with pytest.raises(elmo.ElmoError) as ei:
            elmo.elmo_train_step_chunked(h, X, rowptr, cols, 0.1, 1024, 0, 0, dX)
        assert ei.value.status == 2, f"status {ei.value.status}: {ei.value}"       # ELMO_ENOMEM
        assert "allocate" in str(ei.value)
    finally:
        del hog
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    elmo.elmo_train_step_chunked(h, X, rowptr, cols, 0.1, 1024, 0, 0, dX)
    elmo.elmo_sync_status(h)
    torch.cuda.synchronize()
    h.close()
