"""Pins for the oracle's streams-per-lane layout (format statement, "Streams
per lane": S = 1, 2 or 4 bit streams per lane and tile, symbol pairs dealt to
a lane's streams in turn):

* a hand-derived blob with two streams per lane (tests/golden/tiny_blobs.txt);
* S = 1 writes exactly the one-stream bytes;
* round trips over all 65,536 patterns, and the independent pure-Python reader
  (tests/nwb1_reader.py) decoding S = 2 and 4 blobs;
* the exact size, recomputed stream by stream from the code lengths;
* a planted mistake in the stream assignment fails these pins."""
import os
import struct

import numpy as np
import pytest

import nwb1_reader
from conftest import golden_lines
from lossless_bf16_weight_nwc_b200 import synth


def _case(name):
    for parts in golden_lines("tiny_blobs.txt"):
        if parts[0] == name:
            return dict(p.split("=", 1) for p in parts[1:])
    raise KeyError(name)


def test_hand_derived_two_streams(orc):
    exp = _case("two_streams")
    w = np.array([[0x4020, 0x3FC0, 0x3FC0, 0x4020]], dtype=np.uint16)
    blob = orc.encode(w, streams=int(exp["streams"]))
    h = nwb1_reader.parse(blob.tobytes())
    assert h["streams"] == 2 and struct.unpack_from("<I", blob.tobytes(), 60)[0] == 1
    assert h["total"] == int(exp["total"]) == blob.size and h["tiles_off"] == 512
    assert list(h["index"]) == [int(v) for v in exp["index"].split(",")]
    chunk = blob[512:]
    n = int(exp["nstreams"])
    assert list(chunk[4096:4096 + n]) == [int(exp["stream_bytes"])] * n
    raw = [int(v, 16) for v in exp["raw"].split(",")]
    assert list(chunk[:4]) == raw and not chunk[4:4096].any()
    words = list(np.frombuffer(chunk[4096 + n:4096 + n + 12].tobytes(), dtype="<u4"))
    assert words == [int(v, 16) for v in exp["words"].split(",")]
    assert np.array_equal(orc.decode(blob), w)


def test_one_stream_is_the_plain_layout(orc):
    """The streams entry point with S = 1 writes the one-stream encoder's bytes."""
    import ctypes
    w = synth.matrix(synth.MatrixSpec("w", 77, 1030, "student_t5", 0.015, 0), 3)
    for tile_cols in (64, 512):
        plain = orc.encode(w, tile_cols=tile_cols)
        out = np.zeros(plain.size, dtype=np.uint8)
        size = ctypes.c_int64()
        rc = orc.lib().orc_encode_streams(w.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16)),
                                          77, 1030, 8, tile_cols, 12, 1,
                                          out.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)),
                                          out.size, ctypes.byref(size))
        assert rc == 0 and size.value == plain.size and np.array_equal(out, plain)


@pytest.mark.parametrize("streams", [2, 4])
def test_round_trips_and_reader(orc, streams):
    allp = np.arange(65536, dtype=np.uint16).reshape(256, 256)
    for tile_cols in (64, 128, 256, 512):
        for lmax in (8, 12):
            blob = orc.encode(allp, tile_cols=tile_cols, lmax=lmax, streams=streams)
            assert np.array_equal(orc.decode(blob), allp)
    rng = np.random.default_rng(streams)
    for shape, tile_cols in (((9, 600), 128), ((17, 130), 64), ((3, 513), 512)):
        w = synth.to_bf16_bits(rng.standard_t(3, size=shape) * 0.02)
        blob = orc.encode(w, tile_cols=tile_cols, lmax=12, streams=streams)
        assert np.array_equal(nwb1_reader.decode(blob.tobytes()), w)
        assert np.array_equal(orc.decode(blob), w)


@pytest.mark.parametrize("streams", [1, 2, 4])
def test_exact_size_stream_by_stream(orc, streams):
    rows, cols, tile_cols = 40, 700, 128
    w = synth.matrix(synth.MatrixSpec("w", rows, cols, "normal", 0.02, 0), streams)
    blob = orc.encode(w, tile_cols=tile_cols, lmax=12, streams=streams)
    lens = nwb1_reader.parse(blob.tobytes())["lens"]
    e = ((w.astype(np.int64) >> 7) & 0xFF)
    cnt = np.bincount(e.reshape(-1), minlength=256)
    filler = int(np.argmax(cnt))
    tr, tc = -(-rows // 8), -(-cols // tile_cols)
    full = np.full((8 * tr, tile_cols * tc), filler, dtype=np.int64)
    full[:rows, :cols] = e
    bits = np.array(lens, dtype=np.int64)[full]
    size = -(-(384 + 4 * (tr * tc + 1)) // 256) * 256
    for j in range(tc):
        for i in range(tr):
            block = bits[8 * i:8 * i + 8, j * tile_cols:(j + 1) * tile_cols]
            nbytes = 0
            for t in range(32):
                # Lane t: row t // 4, columns 64 m + 16 (t % 4) + 0..15 of each group m.
                k_bits = block[t // 4].reshape(-1, 4, 16)[:, t % 4, :].reshape(-1)
                for jj in range(streams):
                    mine = [k for k in range(k_bits.size) if (k // 2) % streams == jj]
                    nbytes += -(-int(k_bits[mine].sum()) // 8)
            size += 8 * tile_cols + 32 * streams + -(-nbytes // 16) * 16
    assert blob.size == size


MUTANT = ("pairs dealt by symbol, not by pair",
          "int stream_of(int t, int k, int streams) { return t * streams + (k / 2) % streams; }",
          "int stream_of(int t, int k, int streams) { return t * streams + k % streams; }")


def test_planted_stream_mistake_is_caught(orc, tmp_path):
    name, old, new = MUTANT
    src = orc.source()
    assert src.count(old) == 1
    path = orc.compile_variant(src.replace(old, new), os.path.join(tmp_path, "mutant.so"))
    with orc.use_library(path):
        caught = False
        for check in (lambda: test_hand_derived_two_streams(orc),
                      lambda: test_round_trips_and_reader(orc, 2)):
            try:
                check()
            except Exception:
                caught = True
        assert caught, name
