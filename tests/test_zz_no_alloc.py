"""nwc_gemv_noalloc: the GEMV for callers that may not allocate device memory.

Some hosts own every device allocation and forbid libraries to call cudaMalloc
(inference servers with a fixed pool, plugins inside another framework), and
code being recorded into a CUDA graph must not allocate either.  This entry
point takes its scratch from an array the library defines statically instead
of a caller workspace.  It must give the same results as nwc_gemv, call after
call, although the array keeps whatever the previous call left in it.

This file sorts last so that a run stopping at the first failure has already
run every other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest

from lossless_bf16_weight_nwc_b200 import synth

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lossless_bf16_weight_nwc_b200 import build
    build.build()
    from lossless_bf16_weight_nwc_b200 import _lib
    torch.cuda.set_device(0)
    return _lib


def within_tolerance(y_new, y_ref, w, x):
    """The GEMV tolerance of the parity tests, applied against nwc_gemv."""
    wf = synth.bf16_bits_to_float(w).astype(np.float64)
    xf = synth.bf16_bits_to_float(x).astype(np.float64)
    bound = 1e-2 * np.outer(np.linalg.norm(xf, axis=1), np.linalg.norm(wf, axis=1)) * 2.0 ** -8
    assert (np.abs(y_new.astype(np.float64) - y_ref.astype(np.float64)) <= bound).all()
    rel = np.linalg.norm(y_new - y_ref) / max(np.linalg.norm(y_ref), 1e-300)
    assert rel <= 2e-3


@pytest.mark.parametrize("rows,cols,batch", [(4096, 4096, 1), (1000, 5120, 4), (520, 2048, 8),
                                             (96, 512, 3)])
def test_matches_workspace_gemv_twice(lib, rows, cols, batch):
    spec = synth.MatrixSpec("w", rows, cols, "normal_outliers", 1 / 64, 0)
    w = synth.matrix(spec, 11)
    x = synth.activations(11, batch, cols)
    m = lib.CompressedMatrix.compress(w)
    xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    y_ref = m.gemv(xt).cpu().numpy()
    for _ in range(2):                                  # the array keeps the last call's bytes
        y = torch.full((batch, rows), float("nan"), dtype=torch.float32, device="cuda")
        lib.nwc_gemv_noalloc(m.handle, xt, y, batch)
        torch.cuda.synchronize()
        within_tolerance(y.cpu().numpy(), y_ref, w, x)
    st, word = lib.nwc_get_device_error()
    assert st == 0, hex(word)


def test_rejects_scratch_beyond_limit(lib):
    # An all-zero 8192 x 20480 matrix: 40 column tiles x 8 batch rows x 8192
    # outputs x 4 bytes of partial sums is more than the 8 MiB limit.
    w = np.zeros((8192, 20480), dtype=np.uint16)
    m = lib.CompressedMatrix.compress(w)
    assert lib.nwc_gemv_workspace_size(m.handle, 8) > lib.NWC_NOALLOC_SCRATCH_BYTES
    x = torch.zeros((8, 20480), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((8, 8192), dtype=torch.float32, device="cuda")
    with pytest.raises(lib.NwcError) as err:
        lib.nwc_gemv_noalloc(m.handle, x, y, 8)
    assert err.value.status == lib.NWC_ERR_SCRATCH_LIMIT
    lib.nwc_gemv_noalloc(m.handle, x[:1], y[:1], 1)     # batch 1 fits: 1.3 MiB
    torch.cuda.synchronize()
    assert not y[:1].any()
