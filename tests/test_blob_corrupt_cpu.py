"""Blobs that do not follow the format are refused on the host with
NWC_ERR_CORRUPT (never a crash, a read past the buffer or another status):
every header field set to an inconsistent value, sizes crafted so that the
tile count times the index entry size wraps around 64 bits, truncations, and
seeded random byte changes in the header, code lengths and index."""
import struct

import numpy as np
import pytest

from lossless_bf16_weight_nwc_b200 import synth

CORRUPT = 4

# Byte offset and struct format of each header field (little-endian).
FIELDS = {"magic": (0, "<I"), "version": (4, "<I"), "header_bytes": (8, "<I"), "lmax": (12, "<I"),
          "rows": (16, "<Q"), "cols": (24, "<Q"), "tile_rows": (32, "<I"),
          "tile_cols": (36, "<I"), "tiles_r": (40, "<Q"), "tiles_c": (48, "<Q"),
          "filler": (56, "<I"), "lens_off": (64, "<Q"), "index_off": (72, "<Q"),
          "tiles_off": (80, "<Q"), "total_bytes": (88, "<Q")}


@pytest.fixture(scope="module")
def lib():
    from lossless_bf16_weight_nwc_b200 import build
    build.build()
    from lossless_bf16_weight_nwc_b200 import _lib
    return _lib


@pytest.fixture(scope="module")
def blob(lib):
    w = synth.matrix(synth.MatrixSpec("w", 40, 200, "student_t5", 0.015, 0), 5)
    plan = lib.nwc_plan(w, lmax=12, tile_cols=64)
    b = lib.nwc_compress_host(plan, w)
    lib.nwc_plan_destroy(plan)
    return b


def get(b, name):
    off, fmt = FIELDS[name]
    return struct.unpack_from(fmt, b, off)[0]


def put(b, name, value):
    off, fmt = FIELDS[name]
    b = b.copy()
    struct.pack_into(fmt, b, off, value)
    return b


def refused(lib, b):
    with pytest.raises(lib.NwcError) as e:
        lib.nwc_blob_device_bytes(b)
    assert e.value.status == CORRUPT
    with pytest.raises(lib.NwcError) as e:
        lib.nwc_schedule_describe(b)
    assert e.value.status == CORRUPT


def test_valid_blob_parses(lib, blob):
    assert lib.nwc_blob_device_bytes(blob) > blob.size
    assert get(blob, "tiles_r") == 5 and get(blob, "tiles_c") == 4


@pytest.mark.parametrize("name,value", [
    ("magic", 0x3142574F), ("version", 2), ("header_bytes", 127), ("lmax", 0), ("lmax", 13),
    ("rows", 0), ("rows", 41), ("rows", 1 << 41), ("cols", 0), ("cols", 257), ("tile_rows", 16),
    ("tile_cols", 96), ("tile_cols", 1024), ("tiles_r", 6), ("tiles_c", 3), ("filler", 256),
    ("lens_off", 0), ("index_off", 388), ("tiles_off", 256), ("tiles_off", 1 << 63),
    ("total_bytes", 0), ("total_bytes", 1 << 40)])
def test_header_field_refused(lib, blob, name, value):
    refused(lib, put(blob, name, value))


def test_tile_count_wrapping_64_bits_refused(lib, blob):
    """tiles_r x tiles_c = 2^62 - 1 fits 64 bits, but its index size 4 (tiles + 1)
    is 2^64: wrapped, the tile area would seem to start at byte 512, and only
    the bytes it reads would stop the index walk from running past the
    buffer."""
    tiles_r, tiles_c = (1 << 31) - 1, (1 << 31) + 1
    assert tiles_r * tiles_c == (1 << 62) - 1 and (4 * (tiles_r * tiles_c + 1)) % (1 << 64) == 0
    b = put(blob, "tile_cols", 64)
    b = put(b, "rows", 8 * tiles_r)
    b = put(b, "cols", 64 * tiles_c)
    b = put(b, "tiles_r", tiles_r)
    b = put(b, "tiles_c", tiles_c)
    b = put(b, "tiles_off", 512)
    refused(lib, b)


def test_code_lengths_refused(lib, blob):
    lens = blob[128:384]
    over = blob.copy()
    over[128:384] = np.where(lens > 0, 1, 0)  # Kraft sum above 1
    refused(lib, over)
    long = blob.copy()
    long[128 + int(np.argmax(lens))] = 13     # longer than lmax
    refused(lib, long)
    no_filler = blob.copy()
    no_filler[128 + get(blob, "filler")] = 0  # the filler exponent has no code
    refused(lib, no_filler)


def test_index_refused(lib, blob):
    index = np.frombuffer(blob[384:384 + 4 * 21].tobytes(), dtype=np.uint32)
    for u, value in [(0, 1), (5, index[4]), (5, index[6] + 1), (20, index[20] + 1),
                     (20, index[20] - 1), (7, 0xFFFFFFFF)]:
        b = blob.copy()
        b[384 + 4 * u:388 + 4 * u] = np.frombuffer(np.uint32(value).tobytes(), dtype=np.uint8)
        refused(lib, b)


def test_truncated_refused(lib, blob):
    for n in (0, 1, 127, 128, 383, 384, 400, get(blob, "tiles_off"), blob.size - 16, blob.size - 1):
        refused(lib, blob[:n].copy())
    refused(lib, np.concatenate([blob, np.zeros(16, np.uint8)]))


def test_random_changes_in_the_head(lib, blob):
    """Seeded random byte changes in the header, code lengths and index: the
    blob either still parses (the change hit a byte the format leaves free, or
    kept every rule) or is refused as corrupt; nothing else happens."""
    rng = np.random.default_rng(11)
    head = get(blob, "tiles_off")
    parsed = 0
    for _ in range(400):
        b = blob.copy()
        for pos in rng.integers(0, head, size=int(rng.integers(1, 5))):
            b[pos] = rng.integers(0, 256)
        try:
            dev = lib.nwc_blob_device_bytes(b)
        except lib.NwcError as e:
            assert e.status == CORRUPT
            continue
        parsed += 1
        assert dev >= b.size
        info, cta, bat, ring = lib.nwc_schedule_describe(b)
        assert info["tiles"] == get(b, "tiles_r") * get(b, "tiles_c") == len(ring)
    assert parsed < 400
