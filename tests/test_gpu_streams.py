"""GPU parity with two bit streams per lane (header streams field = 1).

A lane's symbol pairs alternate between its two streams, so its decoder
follows two independent chains.  Every kernel must read the layout: bit-exact
decompression and row gather, and the GEMV within the parity tolerance of the
FP64 oracle on both the CUDA-core and the tensor-core kernel.  Blobs come from
the library's encoder and from the oracle's.
"""
import numpy as np
import pytest

from lossless_bf16_weight_nwc_b200 import synth
from test_gpu_parity import bits, no_device_error, to_bf16, tolerance_check

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


SHAPES = [((8, 512), 512), ((77, 1030), 512), ((1000, 1026), 512), ((129, 300), 256),
          ((40, 200), 128), ((17, 130), 64), ((2048, 4096), 512), ((4100, 96), 512)]


@pytest.mark.parametrize("lmax", [0, 12])
@pytest.mark.parametrize("shape,tile_cols", SHAPES)
def test_two_streams_all_kernels(lib, orc, shape, tile_cols, lmax):
    spec = synth.MatrixSpec("w", shape[0], shape[1], "normal_outliers", 1 / 64, 5)
    w = synth.matrix(spec, 9)
    m = lib.CompressedMatrix.compress(w, tile_cols=tile_cols, lmax=lmax, streams=2)
    assert int(m.image[60:64].cpu().numpy().view(np.uint32)[0]) == 1
    assert np.array_equal(bits(m.decompress()), w)
    rng = np.random.default_rng(1)
    ids = np.concatenate([[0, shape[0] - 1], rng.integers(0, shape[0], 9)]).astype(np.int32)
    assert np.array_equal(bits(m.gather_rows(torch.from_numpy(ids).cuda())), w[ids])
    for batch in (1, 3, 12):                          # CUDA-core kernel
        x = synth.activations(9, batch, spec.cols)
        xt = to_bf16(x)
        assert lib.nwc_gemv_path(m.handle, xt, batch)[1] is False
        tolerance_check(m.gemv(xt).cpu().numpy(), orc.gemv(w, x), w, x)
    if spec.cols % 8 == 0:
        for batch in (1, 33, 64):                     # tensor-core kernel
            lib.nwc_gemv_set_tc_min_batch(m.handle, 1)
            x = synth.activations(9, batch, spec.cols)
            xt = to_bf16(x)
            assert lib.nwc_gemv_path(m.handle, xt, batch) == (1, True)
            tolerance_check(m.gemv(xt).cpu().numpy(), orc.gemv(w, x), w, x)
    no_device_error(lib, m)


@pytest.mark.parametrize("lmax", [7, 12])
def test_two_streams_oracle_blob(lib, orc, lmax):
    spec = synth.MatrixSpec("w", 300, 2000, "student_t5", 0.015, 2)
    w = synth.matrix(spec, 4)
    blob = orc.encode(w, lmax=lmax, streams=2)
    m = lib.CompressedMatrix.from_blob(blob)
    assert np.array_equal(bits(m.decompress()), w)
    x = synth.activations(4, 5, spec.cols)
    tolerance_check(m.gemv(to_bf16(x)).cpu().numpy(), orc.gemv(w, x), w, x)
    no_device_error(lib, m)


def test_two_streams_every_pattern(lib):
    w = np.arange(65536, dtype=np.uint16).reshape(256, 256)
    m = lib.CompressedMatrix.compress(w, streams=2)
    assert np.array_equal(bits(m.decompress()), w)
    no_device_error(lib, m)
