"""Pins for the oracle encoder/decoder against the NWB1 format statement.

* hand-derived tiny blobs (tests/golden/tiny_blobs.txt);
* an independent pure-Python reader (tests/nwb1_reader.py) decodes oracle blobs;
* the exact size invariant, recomputed from the histogram and the code lengths;
* corrupted or truncated blobs are rejected.
"""
import struct

import numpy as np
import pytest

import nwb1_reader
from conftest import golden_lines
from lossless_bf16_weight_nwc_b200 import synth


def _golden_cases():
    out = {}
    for parts in golden_lines("tiny_blobs.txt"):
        out[parts[0]] = dict(p.split("=", 1) for p in parts[1:])
    return out


@pytest.mark.parametrize("case,weights", [("one_weight", [[0x4020]]),
                                          ("two_weights", [[0x4020, 0x3FC0]])])
def test_hand_derived_blobs(orc, case, weights):
    exp = _golden_cases()[case]
    w = np.array(weights, dtype=np.uint16)
    blob = orc.encode(w)
    h = nwb1_reader.parse(blob.tobytes())
    assert h["rows"] == int(exp["rows"]) and h["cols"] == int(exp["cols"])
    assert h["filler"] == int(exp["filler"], 16)
    assert h["total"] == int(exp["total"]) == blob.size
    assert h["tiles_off"] == int(exp["tiles_off"])
    assert list(h["index"]) == [int(v) for v in exp["index"].split(",")]
    assert h["coded_bits"] == int(exp["coded_bits"])
    present = {s: l for s, l in enumerate(h["lens"]) if l}
    assert len(present) == int(exp["nlens"])
    for key, val in exp.items():
        if key.startswith("len["):
            assert present[int(key[4:-1], 16)] == int(val)
    chunk = blob[h["tiles_off"]:]
    assert list(chunk[4096:4096 + 32]) == [int(exp["lane_bytes"])] * 32
    assert chunk[0] == int(exp["raw0"], 16)
    if "raw1" in exp:
        assert chunk[1] == int(exp["raw1"], 16)
        assert not chunk[2:4096].any()
    else:
        assert not chunk[1:4096].any()
    first_word = struct.unpack_from("<I", chunk.tobytes(), 4096 + 32)[0]
    assert first_word == int(exp["stream_first_word"], 16)
    assert np.array_equal(orc.decode(blob), w)
    assert np.array_equal(nwb1_reader.decode(blob.tobytes()), w)


@pytest.mark.parametrize("shape,tile_cols,lmax", [((8, 512), 512, 12), ((9, 513), 512, 12),
                                                  ((17, 200), 64, 8), ((3, 130), 128, 10),
                                                  ((24, 256), 256, 12)])
def test_independent_reader_agrees(orc, shape, tile_cols, lmax):
    rng = np.random.default_rng(shape[0] * 1000 + shape[1])
    w = synth.to_bf16_bits(rng.standard_t(3, size=shape) * 0.02)
    blob = orc.encode(w, tile_cols=tile_cols, lmax=lmax)
    assert np.array_equal(nwb1_reader.decode(blob.tobytes()), w)
    assert np.array_equal(orc.decode(blob), w)


@pytest.mark.parametrize("rows,cols,tile_cols", [(1024, 1024, 512), (100, 1000, 512),
                                                 (64, 700, 128), (7, 5, 64)])
def test_exact_size_invariant(orc, rows, cols, tile_cols):
    """total = header area + lens + index + sum over tiles of
    (raw 8 * tile_cols + 32 + round_up16(sum_lanes ceil(bits_lane / 8))), and the sum
    of all code lengths equals sum_s count(s) * len(s) from the histogram."""
    spec = synth.MatrixSpec("w", rows, cols, "normal", 0.02, 5)
    w = synth.matrix(spec, 9)
    blob = orc.encode(w, tile_cols=tile_cols)
    h = nwb1_reader.parse(blob.tobytes())
    lens = np.array(h["lens"], dtype=np.int64)
    cnt = orc.histogram(w).astype(np.int64)
    tiles_r, tiles_c = -(-rows // 8), -(-cols // tile_cols)
    fillers = tiles_r * 8 * tiles_c * tile_cols - rows * cols
    filler = int(np.argmax(cnt))                        # first maximum = smallest symbol
    assert h["filler"] == filler
    cnt[filler] += fillers
    assert h["coded_bits"] == int((cnt * lens).sum())
    # Recount the lane streams symbol by symbol from the matrix itself.
    padded = np.full((tiles_r * 8, tiles_c * tile_cols), filler, dtype=np.int64)
    padded[:rows, :cols] = (w.astype(np.int64) >> 7) & 0xFF
    area = 0
    for j in range(tiles_c):
        for i in range(tiles_r):
            tile = padded[8 * i:8 * i + 8, tile_cols * j:tile_cols * (j + 1)]
            stream = 0
            for t in range(32):
                # lane t = 4 g + c: row g, columns 64 m + 16 c .. + 15 of each group m
                cols_t = [64 * m + 16 * (t % 4) + kk for m in range(tile_cols // 64)
                          for kk in range(16)]
                bits = int(lens[tile[t // 4, cols_t]].sum())
                stream += -(-bits // 8)
            area += 8 * tile_cols + 32 + -(-stream // 16) * 16
    tiles_off = -(-(128 + 256 + 4 * (tiles_r * tiles_c + 1)) // 256) * 256
    assert blob.size == tiles_off + area


def test_corruption_is_rejected(orc):
    spec = synth.MatrixSpec("w", 16, 1024, "normal", 0.02, 0)
    w = synth.matrix(spec, 1)
    blob = orc.encode(w)
    h = nwb1_reader.parse(blob.tobytes())
    bad = blob.copy()
    bad[0] ^= 1                                            # magic
    with pytest.raises(orc.OracleError):
        orc.decode(bad)
    with pytest.raises(orc.OracleError):                   # truncated
        orc.decode(blob[:-16])
    bad = blob.copy()
    bad[128 + int(np.flatnonzero(np.array(h["lens"]))[0])] = 0   # drop a code
    with pytest.raises(orc.OracleError):
        orc.decode(bad)
    bad = blob.copy()
    struct.pack_into("<I", bad, 384 + 4, h["index"][1] + 1)      # index off by 16 bytes
    with pytest.raises(orc.OracleError):
        orc.decode(bad)
    bad = blob.copy()
    bad[h["tiles_off"] + 4096] += 1                               # lane length
    with pytest.raises(orc.OracleError):
        orc.decode(bad)
