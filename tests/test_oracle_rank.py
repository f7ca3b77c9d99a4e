"""Pins for the oracle's ranked unary code, variant NWR1 ("NWC — Neural Weight
Compression", "How it works > Prefix code instead of rANS", format v9):

* hand-derived tiny blobs (tests/golden/tiny_rank_blobs.txt);
* round trip over all 65,536 BF16 patterns, shuffled, odd shapes, every rank
  count and tile width, and the workload generators;
* the rank table against an independent ordering of the counts;
* the exact code bits and blob size, recomputed lane by lane with numpy from the
  format statement (not from the oracle's code);
* the mean code length equals the closed form of the format-variant study;
* blobs that break the format are refused;
* planted mistakes in copies of the oracle source fail these pins."""
import os
import struct

import numpy as np
import pytest

from conftest import golden_lines
from lossless_bf16_weight_nwc_b200 import synth
from test_format_variants_cpu import unary_rank_cost

CORRUPT = -3


def _header(blob):
    b = blob.tobytes()
    return {"magic": struct.unpack_from("<I", b, 0)[0], "R": struct.unpack_from("<I", b, 12)[0],
            "rows": struct.unpack_from("<Q", b, 16)[0], "cols": struct.unpack_from("<Q", b, 24)[0],
            "tile_cols": struct.unpack_from("<I", b, 36)[0],
            "filler": struct.unpack_from("<I", b, 56)[0],
            "tiles_off": struct.unpack_from("<Q", b, 80)[0],
            "total": struct.unpack_from("<Q", b, 88)[0],
            "code_bits": struct.unpack_from("<Q", b, 96)[0]}


@pytest.mark.parametrize("case", ["one_weight", "escape", "ties"])
def test_hand_derived_rank_blobs(orc, case):
    exp = {p[0]: dict(kv.split("=", 1) for kv in p[1:]) for p in golden_lines("tiny_rank_blobs.txt")}[case]
    w = np.array([[int(v, 16) for v in exp["weights"].split(",")]], dtype=np.uint16)
    blob = orc.rank_encode(w, tile_cols=64, ranks=int(exp["ranks"]))
    h = _header(blob)
    assert h["magic"] == 0x3152574E and h["R"] == int(exp["R"])
    table = [int(v, 16) for v in exp["table"].split(",")]
    assert list(blob[128:128 + len(table)]) == table and not blob[128 + len(table):384].any()
    assert orc.rank_table(w, tile_cols=64, ranks=int(exp["ranks"])) == table
    assert h["filler"] == int(exp["filler"], 16)
    assert h["total"] == int(exp["total"]) == blob.size and h["tiles_off"] == 512
    assert list(np.frombuffer(blob[384:392].tobytes(), dtype=np.uint32)) == \
        [int(v) for v in exp["index"].split(",")]
    assert h["code_bits"] == int(exp["code_bits"])
    chunk = blob[512:]
    raw = [int(v, 16) for v in exp["raw"].split(",")]
    assert list(chunk[:len(raw)]) == raw and not chunk[len(raw):512].any()
    assert list(chunk[512:544]) == [int(exp["lane0_bytes"])] + [4] * 31
    words = list(np.frombuffer(chunk[544:552].tobytes(), dtype="<u4"))
    assert words == [int(v, 16) for v in exp["words"].split(",")]
    assert np.array_equal(orc.rank_decode(blob), w)


def test_every_pattern_round_trips(orc):
    allp = np.arange(65536, dtype=np.uint16).reshape(256, 256)
    for tile_cols in (64, 128, 256, 512):
        for ranks in (1, 2, 7):
            assert np.array_equal(orc.rank_decode(orc.rank_encode(allp, tile_cols, ranks)), allp)
    rng = np.random.default_rng(2)
    shuffled = rng.permutation(allp.reshape(-1)).reshape(128, 512)
    assert np.array_equal(orc.rank_decode(orc.rank_encode(shuffled)), shuffled)
    for shape in ((1, 1), (1, 513), (9, 65), (77, 1030), (4100, 96)):
        w = synth.to_bf16_bits(rng.standard_t(4, size=shape) * 0.02)
        assert np.array_equal(orc.rank_decode(orc.rank_encode(w, tile_cols=128)), w)
    same = np.full((5, 70), 0xBF80, dtype=np.uint16)
    assert np.array_equal(orc.rank_decode(orc.rank_encode(same)), same)


@pytest.mark.parametrize("name", synth.WORKLOADS)
def test_workload_generators_round_trip(orc, name):
    wl = synth.workload(name)
    for spec in wl.matrices[:2]:
        w = synth.matrix(spec, wl.seed, 0, min(spec.rows, 64))
        assert np.array_equal(orc.rank_decode(orc.rank_encode(w)), w)


def _independent_table(w, ranks, tile_cols):
    """Counts of exponent bits 14..8 with the fillers, ordered by count then value."""
    e = (w.astype(np.int64) >> 8) & 0x7F
    cnt = np.bincount(e.reshape(-1), minlength=128)
    filler = int(np.argmax(cnt))                  # first maximum = smallest value
    rows, cols = w.shape
    padded = -(-rows // 8) * 8 * (-(-cols // tile_cols) * tile_cols)
    cnt[filler] += padded - rows * cols
    order = sorted(np.flatnonzero(cnt).tolist(), key=lambda v: (-cnt[v], v))
    return order[:ranks], cnt, filler


@pytest.mark.parametrize("shape,tile_cols,ranks", [((64, 512), 512, 7), ((9, 513), 512, 7),
                                                    ((40, 200), 64, 3), ((17, 130), 128, 1),
                                                    ((256, 256), 256, 7)])
def test_size_and_code_bits_recomputed(orc, shape, tile_cols, ranks):
    rng = np.random.default_rng(shape[0] * 7 + ranks)
    if shape == (256, 256):
        w = np.arange(65536, dtype=np.uint16).reshape(shape)
    else:
        w = synth.to_bf16_bits(rng.standard_t(3, size=shape) * 0.03)
    table, _, filler = _independent_table(w, ranks, tile_cols)
    assert orc.rank_table(w, tile_cols, ranks) == table
    R = len(table)
    rank_of = {v: r for r, v in enumerate(table)}
    rows, cols = shape
    tr, tc = -(-rows // 8), -(-cols // tile_cols)
    e = np.full((tr * 8, tc * tile_cols), filler, dtype=np.int64)
    e[:rows, :cols] = (w.astype(np.int64) >> 8) & 0x7F
    bits = np.vectorize(lambda v: 1 + (rank_of[v] + 1 if v in rank_of else R + 7))(e)
    tiles_off = -(-(384 + 4 * (tr * tc + 1)) // 256) * 256
    size = tiles_off
    for j in range(tc):
        for i in range(tr):
            block = bits[8 * i:8 * i + 8, j * tile_cols:(j + 1) * tile_cols]
            # Lane 4g + c holds row g, columns 64m + 16c .. 64m + 16c + 15 of every group m.
            lane_bytes = [-(-int(block[t // 4].reshape(-1, 4, 16)[:, t % 4, :].sum()) // 8)
                          for t in range(32)]
            size += 8 * tile_cols + 32 + -(-sum(lane_bytes) // 16) * 16
    blob = orc.rank_encode(w, tile_cols, ranks)
    assert blob.size == size
    assert _header(blob)["code_bits"] == int(bits.sum())


def test_mean_code_length_is_the_closed_form(orc):
    """No fillers (a whole number of tiles): the mean code bits per weight are
    the sign bit plus the unary cost of the format-variant study."""
    wl = synth.workload("attn_4096_outliers")
    w = synth.matrix(wl.matrices[0], wl.seed, 0, 256)
    e = (w.astype(np.int64) >> 8) & 0x7F
    cnt = np.bincount(e.reshape(-1), minlength=128)
    blob = orc.rank_encode(w)
    assert _header(blob)["code_bits"] / w.size == pytest.approx(1 + unary_rank_cost(cnt, 7, 7),
                                                                 rel=1e-12)


def test_broken_blobs_refused(orc):
    w = synth.to_bf16_bits(np.random.default_rng(1).normal(0, 0.02, size=(16, 128)))
    blob = orc.rank_encode(w, tile_cols=64)
    assert np.array_equal(orc.rank_decode(blob), w)
    R = _header(blob)["R"]
    cases = []
    def changed(pos, value):
        b = blob.copy()
        b[pos] = value
        return b

    cases = [changed(0, blob[0] ^ 1),           # magic
             changed(12, 0),                    # R = 0
             changed(12, 8),                    # R > 7
             changed(129, blob[128]),           # a repeated rank value
             changed(128 + R, 5),               # bytes after the table
             changed(56, blob[56] ^ 1),         # the filler is not rank 0
             changed(128, 0x80),                # not a 7-bit value
             blob[:-16].copy(),                 # truncated
             changed(blob.size - 1, 0xFF)]      # nonzero stream padding
    for bad in cases:
        with pytest.raises(orc.OracleError) as e:
            orc.rank_decode(bad)
        assert e.value.code == CORRUPT


def test_escape_of_a_ranked_value_refused(orc):
    """A ranked value written as an escape decodes to the right number but is
    not the canonical stream: it is refused.  Built from the 'escape' golden
    case by moving 0x40 into the table (R stays 1): the escape now names it."""
    w = np.array([[0x3F80, 0xBF80, 0x4000]], dtype=np.uint16)
    blob = orc.rank_encode(w, tile_cols=64, ranks=1)
    bad = blob.copy()
    bad[128] = 0x40          # table [0x40]: the filler no longer matches rank 0 ...
    bad[56] = 0x40           # ... so move the filler too; the escape now names 0x40
    with pytest.raises(orc.OracleError):
        orc.rank_decode(bad)


# ---- planted mistakes -------------------------------------------------------

MUTANTS = [
    ("sign after the rank code", "  bits->push_back((uint8_t)sign);\n  int r = 0;",
     "  int r = 0;"),
    ("rank ties to the larger value", "[&](int a, int b) { return cnt[a] > cnt[b]; });",
     "[&](int a, int b) { return cnt[a] > cnt[b] || (cnt[a] == cnt[b] && a > b); });"),
    ("field is exponent bits 13..7", "*e = (w >> 8) & 0x7F;", "*e = (w >> 7) & 0x7F;"),
    ("escape drops the top bit", "for (int b = 6; b >= 0; --b) bits->push_back",
     "for (int b = 5; b >= 0; --b) bits->push_back"),
    ("one rank too many", "const int n = (int)std::min<size_t>(present.size(), (size_t)ranks);",
     "const int n = (int)std::min<size_t>(present.size(), (size_t)ranks + 1);"),
]


def _rank_pins_pass(orc):
    try:
        for case in ("one_weight", "escape", "ties"):
            test_hand_derived_rank_blobs(orc, case)
        allp = np.arange(65536, dtype=np.uint16).reshape(256, 256)
        if not np.array_equal(orc.rank_decode(orc.rank_encode(allp, 64, 7)), allp):
            return False
        test_size_and_code_bits_recomputed(orc, (40, 200), 64, 3)
        return True
    except Exception:
        return False


def test_real_oracle_passes_rank_pins(orc):
    assert _rank_pins_pass(orc)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_rank_mistake_is_caught(orc, tmp_path, name, old, new):
    src = orc.source()
    assert src.count(old) == 1, name
    path = orc.compile_variant(src.replace(old, new), os.path.join(tmp_path, "mutant.so"))
    with orc.use_library(path):
        caught = not _rank_pins_pass(orc)
    assert caught, f"planted mistake not caught: {name}"
