"""The library's host side of the verbatim-run variant NWE1 ("Unweight",
"Compressing BF16 Weights"), on the CPU: its multithreaded encoder writes the
oracle's bytes, the blob parser takes what the kernels read and refuses the
rest, and the plan options select it."""
import ctypes

import numpy as np
import pytest

from lossless_bf16_weight_nwc_b200 import synth

CORRUPT, UNSUPPORTED, INVALID = 4, 2, 1


@pytest.fixture(scope="module")
def lib():
    from lossless_bf16_weight_nwc_b200 import _lib
    return _lib


def _host_blob(lib, w, **kw):
    plan = lib.nwc_plan(w, code=lib.NWC_CODE_ESCAPE, threads=3, **kw)
    try:
        dev_bytes, blob_bytes = lib.nwc_plan_size(plan)
        blob = lib.nwc_compress_host(plan, w)
    finally:
        lib.nwc_plan_destroy(plan)
    assert blob.size == blob_bytes
    return blob, dev_bytes


@pytest.mark.parametrize("shape,tile_cols,keep,lmax,dist", [
    ((1024, 1024), 512, 0, 0, "student_t5"), ((9, 513), 512, 16, 7, "student_t5"),
    ((77, 1030), 256, 4, 0, "normal_outliers"), ((8, 64), 64, 1, 0, "normal"),
    ((333, 200), 128, 16, 6, "normal_outliers"), ((1, 1), 512, 0, 0, "normal"),
    ((40, 4096), 512, 2, 7, "normal_outliers")])
def test_encoder_byte_identical_to_oracle(lib, orc, shape, tile_cols, keep, lmax, dist):
    w = synth.matrix(synth.MatrixSpec("w", shape[0], shape[1], dist, 0.015, 3), 11)
    blob, dev_bytes = _host_blob(lib, w, lmax=lmax, tile_cols=tile_cols, keep=keep)
    ref = orc.escape_encode(w, tile_cols=tile_cols, lmax=lmax or 7, keep=keep or 16)
    assert np.array_equal(blob, ref)
    assert np.array_equal(orc.escape_decode(blob), w)
    # The device image: the blob, the 64 KiB decode table, schedules, scratch.
    assert dev_bytes == lib.nwc_blob_device_bytes(blob) > blob.size + 65536


def test_all_patterns_and_all_runs_verbatim(lib, orc):
    allp = np.arange(65536, dtype=np.uint16).reshape(256, 256)
    for keep in (1, 16, 128):
        blob, dev_bytes = _host_blob(lib, allp, keep=keep)
        assert np.array_equal(blob, orc.escape_encode(allp, keep=keep))
        assert lib.nwc_blob_device_bytes(blob) == dev_bytes
    # Every run verbatim: no code at all, still a valid image.
    w = np.tile(np.array([0x3F80, 0x4000], dtype=np.uint16), (16, 512))
    blob, dev_bytes = _host_blob(lib, w, keep=1)
    assert np.array_equal(blob, orc.escape_encode(w, keep=1)) and not blob[128:384].any()
    assert lib.nwc_blob_device_bytes(blob) == dev_bytes
    info, _, _, ring = lib.nwc_schedule_describe(blob)
    assert info["tiles"] == len(ring) == 4


def test_parser_refuses_what_breaks_the_format(lib, orc):
    w = synth.matrix(synth.MatrixSpec("w", 64, 1024, "normal_outliers", 0.015, 3), 5)
    blob = orc.escape_encode(w, keep=10)             # 10 codes, 234 of 1024 runs verbatim
    lib.nwc_blob_device_bytes(blob)

    def status(b):
        with pytest.raises(lib.NwcError) as e:
            lib.nwc_blob_device_bytes(b)
        return e.value.status

    bad = blob.copy()
    bad[60:64] = 0                                   # K = 0
    assert status(bad) == CORRUPT
    bad = blob.copy()
    bad[60:64] = np.frombuffer(np.uint32(257).tobytes(), np.uint8)
    assert status(bad) == CORRUPT                    # K > 256
    bad = blob.copy()
    bad[60:64] = np.frombuffer(np.uint32(9).tobytes(), np.uint8)
    assert status(bad) == CORRUPT                    # more codes than kept exponents
    bad = blob.copy()
    bad[388:392] = 0                                 # a chunk smaller than raw + flags + lengths
    assert status(bad) == CORRUPT
    # Longer codes are a valid NWE1 blob that no kernel reads.
    assert status(orc.escape_encode(w, lmax=12, keep=10)) == UNSUPPORTED


def test_plan_options(lib):
    w = synth.matrix(synth.MatrixSpec("w", 16, 256, "normal", 0.02, 0), 1)
    for kw, st in (({"keep": 257}, INVALID), ({"lmax": 8}, UNSUPPORTED),
                   ({"streams": 2}, UNSUPPORTED)):
        with pytest.raises(lib.NwcError) as e:
            lib.nwc_plan(w, code=lib.NWC_CODE_ESCAPE, **kw)
        assert e.value.status == st
    # The options layout without `keep` means 16 kept exponents.
    opts = lib.nwc_opts(28, 0, 8, 512, 1, lib.NWC_CODE_ESCAPE, 1)
    plan = ctypes.c_void_p()
    assert lib.LIB.nwc_plan(w.ctypes.data, 16, 256, ctypes.byref(opts), ctypes.byref(plan)) == 0
    blob = lib.nwc_compress_host(plan, w)
    lib.nwc_plan_destroy(plan)
    assert int.from_bytes(blob[:4].tobytes(), "little") == 0x3145574E
    assert int.from_bytes(blob[60:64].tobytes(), "little") == min(16, len(set((w >> 7).ravel() & 0xFF)))
