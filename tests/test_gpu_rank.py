"""GPU parity of the ranked unary code (variant NWR1; "NWC", "How it works >
Prefix code instead of rANS", format v9) against the oracle.

Every kernel reads it with a table-free reader (a code is the sign bit, then
r zeros and a one, or R zeros and the 7-bit field): decompression and row
gather bit-exact against the oracle's rank decoder, and the GEMV within the
parity tolerance on both the CUDA-core and the tensor-core kernel.
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


@pytest.mark.parametrize("ranks", [1, 3, 7])
@pytest.mark.parametrize("shape,tile_cols", SHAPES)
def test_rank_code_all_kernels(lib, orc, shape, tile_cols, ranks):
    spec = synth.MatrixSpec("w", shape[0], shape[1], "normal_outliers", 1 / 64, 6)
    w = synth.matrix(spec, 12)
    m = lib.CompressedMatrix.compress(w, tile_cols=tile_cols, lmax=ranks, code=lib.NWC_CODE_RANK)
    blob = orc.rank_encode(w, tile_cols=tile_cols, ranks=ranks)
    assert np.array_equal(m.image[:blob.size].cpu().numpy(), blob)   # the oracle's bytes
    assert np.array_equal(bits(m.decompress()), orc.rank_decode(blob))
    rng = np.random.default_rng(2)
    ids = np.concatenate([[0, shape[0] - 1], rng.integers(0, shape[0], 9)]).astype(np.int32)
    assert np.array_equal(bits(m.gather_rows(torch.from_numpy(ids).cuda())), w[ids])
    for batch in (1, 3, 12):                          # CUDA-core kernel
        x = synth.activations(12, batch, spec.cols)
        xt = to_bf16(x)
        assert lib.nwc_gemv_path(m.handle, xt, batch)[1] is False
        tolerance_check(m.gemv(xt).cpu().numpy(), orc.gemv(w, x), w, x)
    if spec.cols % 8 == 0:
        lib.nwc_gemv_set_tc_min_batch(m.handle, 1)
        for batch in (1, 33, 64):                     # tensor-core kernel
            x = synth.activations(12, batch, spec.cols)
            xt = to_bf16(x)
            assert lib.nwc_gemv_path(m.handle, xt, batch) == (1, True)
            tolerance_check(m.gemv(xt).cpu().numpy(), orc.gemv(w, x), w, x)
    no_device_error(lib, m)


def test_rank_code_every_pattern_and_oracle_blob(lib, orc):
    """All 65,536 patterns (every value of the 7-bit field, escapes included)
    from the oracle's blob, uploaded and decoded on the GPU."""
    w = np.arange(65536, dtype=np.uint16).reshape(256, 256)
    for ranks in (2, 7):
        blob = orc.rank_encode(w, tile_cols=128, ranks=ranks)
        m = lib.CompressedMatrix.from_blob(blob)
        assert np.array_equal(bits(m.decompress()), w)
        no_device_error(lib, m)
