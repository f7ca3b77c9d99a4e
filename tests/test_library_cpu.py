"""libnwc on the CPU: it loads, exports every symbol include/nwc.h declares, and
its host encoder writes the same bytes as the oracle (no GPU calls here)."""
import re

import numpy as np
import pytest

from conftest import ROOT
from lossless_bf16_weight_nwc_b200 import synth

UNSUPPORTED = 2  # NWC_ERR_UNSUPPORTED


@pytest.fixture(scope="module")
def lib():
    from lossless_bf16_weight_nwc_b200 import build
    build.build()
    from lossless_bf16_weight_nwc_b200 import _lib
    return _lib


def test_exports_every_declared_symbol(lib):
    with open(f"{ROOT}/include/nwc.h") as f:
        text = f.read()
    declared = set(re.findall(r"\b(nwc_[a-z_]+)\s*\(", text))
    assert len(declared) >= 16
    for name in declared:
        assert hasattr(lib.LIB, name), name
    assert set(lib.EXPORTED) == declared


def test_status_strings(lib):
    for code in range(9):
        assert lib.LIB.nwc_status_string(code)


@pytest.mark.parametrize("shape,tile_cols,lmax", [((1024, 1024), 512, 12), ((9, 513), 512, 12),
                                                  ((77, 1030), 256, 10), ((8, 64), 64, 8),
                                                  ((333, 200), 128, 12), ((1, 1), 512, 12)])
def test_host_encoder_byte_identical_to_oracle(lib, orc, shape, tile_cols, lmax):
    spec = synth.MatrixSpec("w", shape[0], shape[1], "student_t5", 0.015, 3)
    w = synth.matrix(spec, 7)
    plan = lib.nwc_plan(w, lmax=lmax, tile_cols=tile_cols, threads=3)
    try:
        dev_bytes, blob_bytes = lib.nwc_plan_size(plan)
        blob = lib.nwc_compress_host(plan, w)
    finally:
        lib.nwc_plan_destroy(plan)
    ref = orc.encode(w, tile_cols=tile_cols, lmax=lmax)
    assert blob.size == blob_bytes == ref.size
    assert np.array_equal(blob, ref)
    assert dev_bytes >= blob_bytes + 16384 and dev_bytes % 256 == 0
    assert lib.nwc_blob_device_bytes(blob) == dev_bytes
    assert np.array_equal(orc.decode(blob), w)


def test_all_patterns_byte_identical(lib, orc):
    w = np.arange(65536, dtype=np.uint16).reshape(256, 256)
    plan = lib.nwc_plan(w, lmax=12)
    blob = lib.nwc_compress_host(plan, w)
    lib.nwc_plan_destroy(plan)
    assert np.array_equal(blob, orc.encode(w))


def test_host_validation(lib):
    w = np.zeros((4, 4), dtype=np.uint16)
    with pytest.raises(lib.NwcError):
        lib.nwc_plan(w, tile_cols=100)
    with pytest.raises(lib.NwcError):
        lib.nwc_plan(w, lmax=13)
    w = (np.arange(256, dtype=np.uint16) << 7).reshape(1, 256)
    with pytest.raises(lib.NwcError):          # 256 exponents do not fit 7-bit codes
        lib.nwc_plan(w, lmax=7)
    bad = np.zeros(512, dtype=np.uint8)
    with pytest.raises(lib.NwcError):
        lib.nwc_blob_device_bytes(bad)


def test_compressed_matrix_checks_tensors_on_the_host(lib, monkeypatch):
    """CompressedMatrix refuses tensors of the wrong type, shape or device before
    any library call (the image lives on the meta device here, so a call that
    got through would fail loudly)."""
    torch = pytest.importorskip("torch")
    monkeypatch.setattr(lib, "nwc_handle_destroy", lambda h: None)
    rows, cols = 24, 40
    m = lib.CompressedMatrix(torch.empty(256, dtype=torch.uint8, device="meta"), object(),
                             rows, cols, 256)
    meta = dict(device="meta")
    with pytest.raises(TypeError):
        m.gemv(torch.zeros((2, cols), dtype=torch.float32, **meta))
    with pytest.raises(ValueError):
        m.gemv(torch.zeros((2, cols + 1), dtype=torch.bfloat16, **meta))
    with pytest.raises(ValueError):   # the host copy of x is not on the matrix's device
        m.gemv(torch.zeros((2, cols), dtype=torch.bfloat16))
    with pytest.raises(ValueError):   # more rows of x than one call takes
        m.gemv(torch.zeros((65, cols), dtype=torch.bfloat16, **meta))
    x = torch.zeros((3, cols), dtype=torch.bfloat16, **meta)
    with pytest.raises(ValueError):
        m.gemv(x, y=torch.zeros((3, rows + 1), dtype=torch.float32, **meta))
    with pytest.raises(TypeError):
        m.gemv(x, y=torch.zeros((3, rows), dtype=torch.bfloat16, **meta))
    with pytest.raises(ValueError):   # pageable host memory is not a valid y
        m.gemv(x, y=torch.zeros((3, rows), dtype=torch.float32))
    with pytest.raises(ValueError):
        m.gemv(x, y=torch.zeros((rows, 3), dtype=torch.float32, **meta).t())
    with pytest.raises(ValueError):
        m.decompress(out=torch.empty((rows, cols + 1), dtype=torch.bfloat16, **meta))
    with pytest.raises(ValueError):
        m.decompress(out=torch.empty((rows, cols), dtype=torch.bfloat16))
    with pytest.raises(TypeError):
        m.decompress(out=torch.empty((rows, cols), dtype=torch.float16, **meta))
    with pytest.raises(TypeError):
        m.gather_rows(torch.zeros(3, dtype=torch.float32))
    empty = m.gather_rows(torch.zeros(0, dtype=torch.int64))
    assert empty.shape == (0, cols) and empty.dtype == torch.bfloat16
    m.handle = None
    with pytest.raises(ValueError):
        m.gemv(x)


@pytest.mark.parametrize("shape,tile_cols,ranks", [((1024, 1024), 512, 0), ((9, 513), 512, 7),
                                                   ((77, 1030), 256, 3), ((8, 64), 64, 1),
                                                   ((333, 200), 128, 7), ((1, 1), 512, 0)])
def test_rank_code_encoder_byte_identical_to_oracle(lib, orc, shape, tile_cols, ranks):
    """The ranked unary code (NWR1): the library's multithreaded host encoder
    writes the oracle's bytes."""
    w = synth.matrix(synth.MatrixSpec("w", shape[0], shape[1], "student_t5", 0.015, 3), 11)
    plan = lib.nwc_plan(w, lmax=ranks, tile_cols=tile_cols, threads=3, code=lib.NWC_CODE_RANK)
    try:
        dev_bytes, blob_bytes = lib.nwc_plan_size(plan)
        blob = lib.nwc_compress_host(plan, w)
    finally:
        lib.nwc_plan_destroy(plan)
    ref = orc.rank_encode(w, tile_cols=tile_cols, ranks=ranks or 7)
    assert blob.size == blob_bytes == ref.size
    assert np.array_equal(blob, ref)
    assert np.array_equal(orc.rank_decode(blob), w)
    # The device image: the blob, the 256-byte rank table, schedules, scratch.
    assert dev_bytes == lib.nwc_blob_device_bytes(blob) > blob.size


def test_rank_code_all_patterns_and_device_image(lib, orc):
    w = np.arange(65536, dtype=np.uint16).reshape(256, 256)
    plan = lib.nwc_plan(w, code=lib.NWC_CODE_RANK)
    blob = lib.nwc_compress_host(plan, w)
    dev_bytes, _ = lib.nwc_plan_size(plan)
    lib.nwc_plan_destroy(plan)
    assert np.array_equal(blob, orc.rank_encode(w))
    assert lib.nwc_blob_device_bytes(blob) == dev_bytes
    info, _, _, ring = lib.nwc_schedule_describe(blob)
    assert info["tiles"] == len(ring) == 32
    # A broken rank table is refused: a repeated ranked value, a value past 127.
    for at, v in ((129, blob[128]), (128, 200)):
        bad = blob.copy()
        bad[at] = v
        with pytest.raises(lib.NwcError) as e:
            lib.nwc_blob_device_bytes(bad)
        assert e.value.status == 4                    # NWC_ERR_CORRUPT


def test_plan_options_code_field(lib):
    import ctypes
    w = synth.matrix(synth.MatrixSpec("w", 16, 256, "normal", 0.02, 0), 1)
    with pytest.raises(lib.NwcError):
        lib.nwc_plan(w, code=3)
    with pytest.raises(lib.NwcError):                   # at most 7 ranks
        lib.nwc_plan(w, lmax=8, code=lib.NWC_CODE_RANK)
    # The options layout without `code` still means the prefix code.
    opts = lib.nwc_opts(20, 0, 8, 512, 1, 1)
    plan = ctypes.c_void_p()
    assert lib.LIB.nwc_plan(w.ctypes.data, 16, 256, ctypes.byref(opts), ctypes.byref(plan)) == 0
    blob = lib.nwc_compress_host(plan, w)
    lib.nwc_plan_destroy(plan)
    assert int.from_bytes(blob[:4].tobytes(), "little") == 0x3142574E
    opts = lib.nwc_opts(16, 0, 8, 512, 1, 0)            # too short for `threads`
    assert lib.LIB.nwc_plan(w.ctypes.data, 16, 256, ctypes.byref(opts), ctypes.byref(plan)) == 1


def test_four_stream_blobs_refused(lib, orc):
    """The format defines 1, 2 or 4 bit streams per lane; the kernels read 1 and
    2, so a device image exists for those and a 4-stream blob is refused."""
    w = synth.matrix(synth.MatrixSpec("w", 40, 600, "normal", 0.02, 0), 2)
    assert lib.nwc_blob_device_bytes(orc.encode(w, tile_cols=128, streams=2)) > 0
    blob = orc.encode(w, tile_cols=128, streams=4)
    with pytest.raises(lib.NwcError) as e:
        lib.nwc_blob_device_bytes(blob)
    assert e.value.status == UNSUPPORTED
    bad = orc.encode(w, tile_cols=128).copy()
    bad[60] = 2                                          # S = 3 is not a layout
    with pytest.raises(lib.NwcError) as e:
        lib.nwc_blob_device_bytes(bad)
    assert e.value.status == 4                           # NWC_ERR_CORRUPT


def test_streams_per_lane_encoder_and_refusals(lib, orc):
    import ctypes
    w = synth.matrix(synth.MatrixSpec("w", 40, 600, "normal", 0.02, 0), 2)
    for streams in (2, 4):
        plan = lib.nwc_plan(w, tile_cols=128, streams=streams)
        dev_bytes, _ = lib.nwc_plan_size(plan)
        blob = lib.nwc_compress_host(plan, w)
        assert np.array_equal(blob, orc.encode(w, tile_cols=128, lmax=7, streams=streams))
        if streams == 2:
            assert dev_bytes == lib.nwc_blob_device_bytes(blob) > blob.size
        else:
            assert dev_bytes == 0
            h = ctypes.c_void_p()
            st = lib.LIB.nwc_compress(plan, w.ctypes.data, 1 << 20, 1 << 30, None,
                                      ctypes.byref(h))
            assert st == UNSUPPORTED and not h.value
        lib.nwc_plan_destroy(plan)
    with pytest.raises(lib.NwcError) as e:
        lib.nwc_plan(w, streams=3)
    assert e.value.status == 1                         # NWC_ERR_INVALID_ARG
    with pytest.raises(lib.NwcError) as e:
        lib.nwc_plan(w, streams=2, code=lib.NWC_CODE_RANK)
    assert e.value.status == UNSUPPORTED
