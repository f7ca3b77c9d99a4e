"""GPU parity of the verbatim-run variant NWE1 ("Unweight", "Compressing BF16
Weights": the most common exponents Huffman-coded, a row of 64 weights that
holds any other exponent stored whole) against the oracle.

Every kernel reads it: a lane's 16 symbols of a run come either from its bit
stream (the 14-bit table) or, when the tile's flag says the run is verbatim,
from the run's exponent bytes in the chunk.  Decompression and row gather are
bit-exact against the oracle's decoder; the GEMV is within the parity
tolerance on both the CUDA-core and the tensor-core kernel, with few, many and
all runs verbatim.
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


def _verbatim_runs(blob):
    return int.from_bytes(blob[104:112].tobytes(), "little")


@pytest.mark.parametrize("keep", [1, 10, 16])
@pytest.mark.parametrize("shape,tile_cols", SHAPES)
def test_escape_all_kernels(lib, orc, shape, tile_cols, keep):
    spec = synth.MatrixSpec("w", shape[0], shape[1], "normal_outliers", 1 / 64, 6)
    w = synth.matrix(spec, 12)
    m = lib.CompressedMatrix.compress(w, tile_cols=tile_cols, code=lib.NWC_CODE_ESCAPE,
                                      keep=keep)
    blob = orc.escape_encode(w, tile_cols=tile_cols, lmax=7, keep=keep)
    assert np.array_equal(m.image[:blob.size].cpu().numpy(), blob)   # the oracle's bytes
    runs = w.shape[0] * -(-w.shape[1] // 64)
    if keep == 1:
        assert _verbatim_runs(blob) >= 0.9 * runs
    assert np.array_equal(bits(m.decompress()), orc.escape_decode(blob))
    rng = np.random.default_rng(2)
    ids = np.concatenate([[0, shape[0] - 1], rng.integers(0, shape[0], 9)]).astype(np.int32)
    assert np.array_equal(bits(m.gather_rows(torch.from_numpy(ids).cuda())), w[ids])
    for batch in (1, 3, 12, 16):                      # CUDA-core kernel
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


def test_escape_every_pattern_and_oracle_blob(lib, orc):
    """All 65,536 patterns from the oracle's blob, uploaded, decoded and
    gathered on the GPU, with 1, 16 and 128 kept exponents."""
    w = np.arange(65536, dtype=np.uint16).reshape(256, 256)
    for keep, tile_cols in ((1, 64), (16, 128), (128, 512)):
        blob = orc.escape_encode(w, tile_cols=tile_cols, lmax=7, keep=keep)
        m = lib.CompressedMatrix.from_blob(blob)
        assert np.array_equal(bits(m.decompress()), w)
        ids = torch.arange(0, 256, 5, dtype=torch.int32, device="cuda")
        assert np.array_equal(bits(m.gather_rows(ids)), w[::5])
        no_device_error(lib, m)


def test_escape_every_run_verbatim(lib, orc):
    """No code at all: every run of every tile is read from the chunk."""
    w = np.tile(np.array([0x3F80, 0x4000], dtype=np.uint16), (64, 2048))   # 64 x 4096
    m = lib.CompressedMatrix.compress(w, code=lib.NWC_CODE_ESCAPE, keep=1)
    assert np.array_equal(bits(m.decompress()), w)
    # A handle made from a copy of the device image alone.
    c = lib.CompressedMatrix(m.image.clone(), None, w.shape[0], w.shape[1], m.blob_bytes)
    c.handle = lib.nwc_handle_from_device(c.image, c.image.numel())
    assert np.array_equal(bits(c.decompress()), w)
    no_device_error(lib, c)
    c.close()
    for batch in (1, 16, 64):
        x = synth.activations(3, batch, w.shape[1])
        lib.nwc_gemv_set_tc_min_batch(m.handle, 17)
        tolerance_check(m.gemv(to_bf16(x)).cpu().numpy(), orc.gemv(w, x), w, x)
    no_device_error(lib, m)


@pytest.mark.parametrize("batch", [1, 64])
def test_escape_llama_shapes_full_size(lib, orc, batch):
    """The Llama-3.1-8B-shaped stack's layer shapes at full size with the
    default 16 kept exponents, sampled rows against the oracle."""
    wl, layer0, _, _ = synth.stack_parts("llama31_8b_stack")
    seen = set()
    for spec in layer0:
        if (spec.rows, spec.cols) in seen:
            continue
        seen.add((spec.rows, spec.cols))
        w = synth.matrix(spec, wl.seed)
        m = lib.CompressedMatrix.compress(w, code=lib.NWC_CODE_ESCAPE)
        x = synth.activations(wl.seed, batch, spec.cols)
        xt = to_bf16(x)
        assert lib.nwc_gemv_path(m.handle, xt, batch)[1] is (batch >= 17)
        y = m.gemv(xt).cpu().numpy()
        idx = np.unique(np.concatenate([np.linspace(0, spec.rows - 1, 256).astype(np.int64),
                                        np.arange(0, 64), np.arange(spec.rows - 64, spec.rows)]))
        tolerance_check(y[:, idx], orc.gemv(w[idx], x), w[idx], x)
        no_device_error(lib, m)
        m.close()


def test_escape_corrupt_flag_field_reported(lib, orc):
    """A flag naming a 64-column group past the tile (tiles of 256 columns have
    four) is caught by the kernels' own check: decompression and gather set the
    handle's corrupt bit and read nothing outside their buffers."""
    spec = synth.MatrixSpec("w", 64, 1024, "normal_outliers", 1 / 64, 6)
    w = synth.matrix(spec, 12)
    blob = orc.escape_encode(w, tile_cols=256, lmax=7, keep=10)
    tiles_off = int.from_bytes(blob[80:88].tobytes(), "little")
    first = int.from_bytes(blob[384:388].tobytes(), "little")
    bad = blob.copy()
    bad[tiles_off + 16 * first + 8 * 256] |= 0x20         # tile 0, row 0, group 5
    for op in ("decompress", "gather"):
        m = lib.CompressedMatrix.from_blob(bad)
        if op == "decompress":
            m.decompress()
        else:
            m.gather_rows(torch.tensor([0, 1], dtype=torch.int32, device="cuda"))
        st, word = m.device_error()
        assert st != 0 and word & 2, (op, st, word)
        m.close()
    m = lib.CompressedMatrix.from_blob(blob)               # the image itself is fine
    assert np.array_equal(bits(m.decompress()), w)
    no_device_error(lib, m)
