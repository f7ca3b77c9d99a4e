"""nwc_gemv_noalloc: the GEMV whose split-K scratch is a static array of the library.

Some hosts own every device allocation and forbid libraries to call cudaMalloc
(inference servers with a fixed pool, plugins inside another framework), and
code being recorded into a CUDA graph must not allocate either.  This entry
point allocates nothing: its scratch is an array the library defines
statically, shared by every call, which keeps whatever the previous call left
in it.  It must give the oracle's result within the GEMV tolerance, and the
same bits as nwc_gemv (the same kernels and the same fixed summation order),
call after call, even when the previous call left other partial sums behind.

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


def to_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def within_tolerance(y_gpu, y_ref, w, x):
    """The parity tests' GEMV tolerance against the FP64 oracle."""
    wf = synth.bf16_bits_to_float(w).astype(np.float64)
    xf = synth.bf16_bits_to_float(x).astype(np.float64)
    bound = 1e-2 * np.outer(np.linalg.norm(xf, axis=1), np.linalg.norm(wf, axis=1)) * 2.0 ** -8
    assert (np.abs(y_gpu.astype(np.float64) - y_ref) <= bound).all()
    rel = np.linalg.norm(y_gpu - y_ref) / max(np.linalg.norm(y_ref), 1e-300)
    assert rel <= 2e-3


@pytest.mark.parametrize("rows,cols,batch", [(4096, 4096, 1), (1000, 5120, 4), (520, 2048, 8),
                                             (96, 512, 3), (700, 3072, 16)])
def test_matches_oracle_and_gemv_twice(lib, orc, rows, cols, batch):
    spec = synth.MatrixSpec("w", rows, cols, "normal_outliers", 1 / 64, 0)
    w = synth.matrix(spec, 11)
    x = synth.activations(11, batch, cols)
    m = lib.CompressedMatrix.compress(w)
    xt = to_bf16(x)
    y_ref = orc.gemv(w, x)
    y_gemv = m.gemv(xt).cpu().numpy()
    # Another matrix and x, so that the shared array holds other partial sums
    # and counters before each checked call.
    other_spec = synth.MatrixSpec("v", rows, cols, "normal", 0.02, 1)
    other = lib.CompressedMatrix.compress(synth.matrix(other_spec, 12))
    ox = to_bf16(synth.activations(12, batch, cols))
    oy = torch.empty((batch, rows), dtype=torch.float32, device="cuda")
    for _ in range(2):
        lib.nwc_gemv_noalloc(other.handle, ox, oy, batch)
        y = torch.full((batch, rows), float("nan"), dtype=torch.float32, device="cuda")
        lib.nwc_gemv_noalloc(m.handle, xt, y, batch)
        torch.cuda.synchronize()
        got = y.cpu().numpy()
        within_tolerance(got, y_ref, w, x)
        assert np.array_equal(got.view(np.uint32), y_gemv.view(np.uint32))
    for mat in (m, other):
        st, word = mat.device_error()
        assert st == 0, hex(word)


def test_rejects_scratch_beyond_limit(lib):
    # An all-zero 8192 x 20480 matrix: 40 column tiles x 8 batch rows x 8192
    # outputs x 4 bytes of partial sums is more than the 8 MiB limit.
    w = np.zeros((8192, 20480), dtype=np.uint16)
    m = lib.CompressedMatrix.compress(w)
    assert lib.nwc_gemv_scratch_bytes(m.handle, 8) > lib.NWC_NOALLOC_SCRATCH_BYTES
    x = torch.zeros((8, 20480), dtype=torch.bfloat16, device="cuda")
    y = torch.full((8, 8192), float("nan"), dtype=torch.float32, device="cuda")
    with pytest.raises(lib.NwcError) as err:
        lib.nwc_gemv_noalloc(m.handle, x, y, 8)
    assert err.value.status == lib.NWC_ERR_SCRATCH_LIMIT
    torch.cuda.synchronize()
    assert torch.isnan(y).all()                          # nothing was launched
    lib.nwc_gemv_noalloc(m.handle, x[:1], y[:1], 1)     # batch 1 fits: 1.3 MiB
    torch.cuda.synchronize()
    assert torch.equal(y[:1], torch.zeros_like(y[:1]))
    st, word = m.device_error()
    assert st == 0, hex(word)
