"""The give-up path of the kernels' bounded waits, made to run on purpose.

Every wait of the kernels on an mbarrier (or on the producer's progress) polls
a bounded number of times, then sets bit 1 of the handle's error word and lets
the CTA leave.  To make one run out without faulting or hanging anything, the
test rewrites one entry of the launch schedule in the device image: CTA 0's
second copy is told to wait for its own release before it is issued.  Nothing
can release it, so the producer's wait on that "empty" barrier gives up with
no copy of that batch in flight, and the consumers waiting for the batch give
up too.  The poll limit is lowered for the test (nwc_test_set_wait_limit) so
that this takes milliseconds.  Afterwards the schedule is rewritten and an
ordinary GEMV on the same device must meet the parity tolerance.
"""
import time

import numpy as np
import pytest

from lossless_bf16_weight_nwc_b200 import synth
from test_gpu_parity import no_device_error, to_bf16, tolerance_check

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")

KSLOTS_CTAS = 256


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lossless_bf16_weight_nwc_b200 import build
    build.build()
    from lossless_bf16_weight_nwc_b200 import _lib
    torch.cuda.set_device(0)
    return _lib


def r256(v):
    return (v + 255) // 256 * 256


def corrupt_need(image, sched_class_off, batch=1):
    """Make batch `batch` of CTA 0 wait for releases up to and including
    itself: its `need` field (u32 3 of its 16-byte descriptor)."""
    batch_off = (4 * (KSLOTS_CTAS + 1) + 15) // 16 * 16
    at = sched_class_off + batch_off + 16 * batch + 12
    image[at:at + 4] = torch.tensor([batch + 1], dtype=torch.int32).view(torch.uint8).to(image.device)


def layout(lib, m, rows_of_x):
    """Offsets of the class-0 schedule and of the tensor-core schedule for
    rows_of_x rows (one per accumulator width: 16, 32, 64 columns)."""
    info = lib.nwc_handle_info(m.handle)
    lmax = int(m.image[12:16].cpu().numpy().view(np.uint32)[0])
    tiles = (m.rows + 7) // 8 * ((m.cols + 511) // 512)
    table = 65536 if lmax <= 7 else 16384
    sched = r256(r256(info["blob_bytes"]) + table)
    batch_off = (4 * (KSLOTS_CTAS + 1) + 15) // 16 * 16
    class_bytes = r256(batch_off + 16 * ((tiles + 1) // 2 + KSLOTS_CTAS) + 4 * tiles)
    tc_bytes = r256(batch_off + 16 * (tiles + KSLOTS_CTAS) + 8 * tiles)
    tc_class = 0 if rows_of_x <= 16 else 1 if rows_of_x <= 32 else 2
    return sched, sched + 2 * class_bytes + tc_class * tc_bytes


@pytest.mark.parametrize("batch", [1, 32])
def test_bounded_wait_gives_up_and_device_recovers(lib, orc, batch):
    spec = synth.MatrixSpec("w", 4096, 4096, "normal", 0.02, 0)
    w = synth.matrix(spec, 31)
    x = synth.activations(31, batch, spec.cols)
    m = lib.CompressedMatrix.compress(w)
    xt = to_bf16(x)
    launches, tc = lib.nwc_gemv_path(m.handle, xt, batch)
    assert tc == (batch >= 17)
    class0, tc_off = layout(lib, m, batch)
    torch.cuda.synchronize()
    corrupt_need(m.image, tc_off if tc else class0)
    y = torch.zeros((batch, spec.rows), dtype=torch.float32, device="cuda")
    lib.nwc_test_set_wait_limit(4096)
    try:
        t0 = time.perf_counter()
        lib.nwc_gemv(m.handle, xt, y, batch)
        torch.cuda.synchronize()
        elapsed = time.perf_counter() - t0
    finally:
        lib.nwc_test_set_wait_limit(0)
    st, word = m.device_error()
    assert st == 6 and word & 1, (st, word)          # NWC_ERR_DEVICE_TIMEOUT
    assert elapsed < 5.0, elapsed
    # A fresh handle on the same image rewrites its schedules (and clears the
    # scratch); the GEMV that follows is ordinary.
    h2 = lib.nwc_handle_from_device(m.image, m.image.numel())
    try:
        lib.nwc_gemv_set_tc_min_batch(h2, 17)
        y2 = torch.full((batch, spec.rows), float("nan"), dtype=torch.float32, device="cuda")
        lib.nwc_gemv(h2, xt, y2, batch)
        torch.cuda.synchronize()
        tolerance_check(y2.cpu().numpy(), orc.gemv(w, x), w, x)
        no_device_error(lib, h2)
    finally:
        lib.nwc_handle_destroy(h2)
    m.close()
