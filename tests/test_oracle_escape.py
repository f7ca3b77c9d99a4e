"""Pins for the oracle's verbatim-run variant NWE1 ("Unweight", "Compressing
BF16 Weights": the most common exponents Huffman-coded, a row of 64 weights
holding any other exponent stored verbatim):

* hand-derived tiny blobs (tests/golden/tiny_escape_blobs.txt);
* with every symbol kept, the blob is NWB1's with a zero flag field in each
  chunk: the coded part is pinned to the NWB1 oracle's pins;
* the escaped runs, the code bits and the exact blob size, recomputed with numpy
  from the format statement (not from the oracle's code);
* the bits per weight equal the costing of the format-variant study;
* a matrix whose every run is escaped has the closed-form size;
* an independent pure-Python reader (tests/nwb1_reader.py) decodes the blobs;
* round trip over all 65,536 BF16 patterns, odd shapes, every tile width and
  kept count, and the workload generators;
* blobs that break the format are refused;
* planted mistakes in copies of the oracle source fail these pins."""
import os
import struct

import numpy as np
import pytest

from conftest import golden_lines
from lossless_bf16_weight_nwc_b200 import synth
from test_format_variants_cpu import escape_rows_cost

CORRUPT = -3


def _u32(blob, off):
    return struct.unpack_from("<I", blob.tobytes(), off)[0]


def _u64(blob, off):
    return struct.unpack_from("<Q", blob.tobytes(), off)[0]


def _bytes(spec):
    """'7f*3,80' -> [0x7f, 0x7f, 0x7f, 0x80]; '-' -> []."""
    out = []
    if spec == "-":
        return out
    for item in spec.split(","):
        v, _, n = item.partition("*")
        out += [int(v, 16)] * (int(n) if n else 1)
    return out


def _counts(spec):
    out = []
    for item in spec.split(","):
        v, _, n = item.partition("*")
        out += [int(v)] * (int(n) if n else 1)
    return out


def _golden(case):
    return {p[0]: dict(kv.split("=", 1) for kv in p[1:])
            for p in golden_lines("tiny_escape_blobs.txt")}[case]


def _golden_matrix(exp):
    rows, cols = (int(v) for v in exp["shape"].split(","))
    w = np.full((rows, cols), int(exp["base"], 16), dtype=np.uint16)
    for item in exp["set"].split(","):
        r, c, v = item.split(":")
        w[int(r), int(c)] = int(v, 16)
    return w


@pytest.mark.parametrize("case", ["all_kept", "one_run", "two_runs", "tie_keep"])
def test_hand_derived_escape_blobs(orc, case):
    exp = _golden(case)
    w = _golden_matrix(exp)
    tile_cols = int(exp["tile_cols"])
    blob = orc.escape_encode(w, tile_cols=tile_cols, lmax=int(exp["lmax"]), keep=int(exp["keep"]))
    assert _u32(blob, 0) == 0x3145574E and _u32(blob, 12) == int(exp["lmax"])
    assert _u32(blob, 56) == int(exp["filler"], 16) and _u32(blob, 60) == int(exp["K"])
    assert _u64(blob, 80) == 512 and _u64(blob, 88) == int(exp["total"]) == blob.size
    assert _u64(blob, 96) == int(exp["code_bits"]) and _u64(blob, 104) == int(exp["n_esc"])
    lens = np.zeros(256, dtype=np.uint8)
    for item in exp["lens"].split(","):
        s, ln = item.split(":")
        lens[int(s, 16)] = int(ln)
    assert np.array_equal(blob[128:384], lens)
    assert list(np.frombuffer(blob[384:392].tobytes(), dtype=np.uint32)) == \
        [int(v) for v in exp["index"].split(",")]
    chunk = blob[512:]
    raw_n = 8 * tile_cols
    raw = np.zeros(raw_n, dtype=np.uint8)
    if exp["raw"] != "-":
        for item in exp["raw"].split(","):
            pos, v = item.split(":")
            raw[int(pos)] = int(v, 16)
    assert np.array_equal(chunk[:raw_n], raw)
    flags = _bytes(exp["flags"])
    assert list(chunk[raw_n:raw_n + 16]) == flags
    runs = _bytes(exp["runs"])
    at = raw_n + 16
    assert list(chunk[at:at + len(runs)]) == runs
    at += len(runs)
    assert list(chunk[at:at + 32]) == _counts(exp["lane_bytes"])
    words = [int(v, 16) for v in exp["words"].split(",")]
    got = list(np.frombuffer(chunk[at + 32:at + 32 + 4 * len(words)].tobytes(), dtype="<u4"))
    assert got == words
    assert np.array_equal(orc.escape_decode(blob), w)


def test_every_symbol_kept_is_nwb1_with_a_flag_field(orc):
    """keep = 256: no run is escaped, the code is NWB1's, and each chunk is the
    NWB1 chunk with 16 zero bytes after the raw plane."""
    rng = np.random.default_rng(11)
    for shape, tile_cols, lmax in (((9, 65), 64, 12), ((40, 700), 256, 12), ((16, 1024), 512, 7)):
        w = synth.to_bf16_bits(rng.standard_normal(shape) * 0.02)
        e = orc.escape_encode(w, tile_cols=tile_cols, lmax=lmax, keep=256)
        b = orc.encode(w, tile_cols=tile_cols, lmax=lmax)
        assert _u64(e, 104) == 0
        for off in (12, 16, 24, 32, 36, 40, 48, 56, 96):
            assert e[off:off + 8].tobytes() == b[off:off + 8].tobytes() or off in (56,) and \
                _u32(e, 56) == _u32(b, 56)
        assert np.array_equal(e[128:384], b[128:384])
        tiles = _u64(b, 40) * _u64(b, 48)
        ie = np.frombuffer(e[384:384 + 4 * (tiles + 1)].tobytes(), dtype="<u4")
        ib = np.frombuffer(b[384:384 + 4 * (tiles + 1)].tobytes(), dtype="<u4")
        assert np.array_equal(ie, ib + np.arange(tiles + 1))        # one more 16-byte unit a tile
        te, tb = _u64(e, 80), _u64(b, 80)
        raw_n = 8 * tile_cols
        for u in range(tiles):
            ce = e[te + 16 * ie[u]:te + 16 * ie[u + 1]]
            cb = b[tb + 16 * ib[u]:tb + 16 * ib[u + 1]]
            assert np.array_equal(ce[:raw_n], cb[:raw_n]) and not ce[raw_n:raw_n + 16].any()
            assert np.array_equal(ce[raw_n + 16:], cb[raw_n:])


def _recompute(orc, w, tile_cols, keep, lmax):
    """Escaped runs, code bits and blob size from the format statement, numpy only
    (code lengths from the pinned package-merge)."""
    rows, cols = w.shape
    tr, tcn, cp = -(-rows // 8), -(-cols // tile_cols), tile_cols // 64
    s = ((w.astype(np.int64) >> 7) & 0xFF)
    filler = int(np.argmax(np.bincount(s.reshape(-1), minlength=256)))
    full = np.full((tr * 8, tcn * tile_cols), filler, dtype=np.int64)
    full[:rows, :cols] = s
    cnt = np.bincount(full.reshape(-1), minlength=256)
    order = sorted(range(256), key=lambda v: (-cnt[v], v))
    kept = np.zeros(256, dtype=bool)
    kept[[v for v in order[:keep] if cnt[v] > 0]] = True
    runs = full.reshape(tr * 8, tcn * cp, 64)
    esc = ~kept[runs].all(axis=2)
    ccnt = np.bincount(runs[~esc].reshape(-1), minlength=256).astype(np.uint64)
    lens = orc.code_lengths(ccnt, lmax) if ccnt.sum() else np.zeros(256, dtype=np.uint8)
    code_bits = int((ccnt * lens.astype(np.uint64)).sum())
    lane_bits = lens[runs].astype(np.int64).reshape(tr * 8, tcn * cp, 4, 16).sum(axis=3)
    lane_bits *= ~esc[:, :, None]
    lane_bits = lane_bits.reshape(tr, 8, tcn, cp, 4).sum(axis=3)        # [tr, g, tcn, c]
    stream = ((lane_bits + 7) // 8).sum(axis=(1, 3))                      # [tr, tcn]
    n_esc = esc.reshape(tr, 8, tcn, cp).sum(axis=(1, 3))
    chunk = 8 * tile_cols + 16 + 64 * n_esc + 32 + (stream + 15) // 16 * 16
    tiles_off = -(-(384 + 4 * (tr * tcn + 1)) // 256) * 256
    return {"size": int(tiles_off + chunk.sum()), "code_bits": code_bits,
            "n_esc": int(esc.sum()), "esc": esc, "K": int(kept.sum()), "cp": cp,
            "tiles_r": tr}


@pytest.mark.parametrize("shape,tile_cols,keep,lmax", [
    ((40, 200), 64, 3, 7), ((77, 1030), 128, 16, 7), ((9, 513), 512, 4, 12),
    ((64, 1024), 256, 1, 7), ((128, 512), 512, 16, 12)])
def test_size_runs_and_code_bits_recomputed(orc, shape, tile_cols, keep, lmax):
    rng = np.random.default_rng(sum(shape) + keep)
    w = synth.to_bf16_bits(rng.standard_t(3, size=shape) * 0.02)
    blob = orc.escape_encode(w, tile_cols=tile_cols, lmax=lmax, keep=keep)
    ref = _recompute(orc, w, tile_cols, keep, lmax)
    assert blob.size == ref["size"]
    assert _u64(blob, 96) == ref["code_bits"] and _u64(blob, 104) == ref["n_esc"]
    assert _u32(blob, 60) == ref["K"]
    # Each chunk's flags name exactly the tile's escaped runs.
    tr, cp = ref["tiles_r"], ref["cp"]
    tiles = tr * -(-shape[1] // tile_cols)
    index = np.frombuffer(blob[384:384 + 4 * (tiles + 1)].tobytes(), dtype="<u4")
    base = _u64(blob, 80)
    for u in range(tiles):
        i, j = u % tr, u // tr
        fl = blob[base + 16 * index[u] + 8 * tile_cols:][:16]
        want = ref["esc"][8 * i:8 * i + 8, cp * j:cp * j + cp]
        got = np.array([[(fl[g] >> m) & 1 for m in range(cp)] for g in range(8)], dtype=bool)
        assert np.array_equal(got, want) and not fl[8:].any()
    assert np.array_equal(orc.escape_decode(blob), w)


@pytest.mark.parametrize("name", ["single_1024", "attn_4096_outliers", "mlp_pair_t5"])
def test_bits_per_weight_match_the_variant_costing(orc, name):
    """Shapes without fillers: coded bits + 8 raw bits per coded weight + 16 bits per
    escaped weight + one flag bit per run is the study's figure exactly."""
    wl = synth.workload(name)
    spec = wl.matrices[0]
    w = synth.matrix(spec, wl.seed, 0, 256).reshape(256, spec.cols)
    for lmax in (7, 12):
        blob = orc.escape_encode(w, tile_cols=512, lmax=lmax, keep=16)
        n, runs = w.size, w.size // 64
        esc = _u64(blob, 104)
        bits = _u64(blob, 96) + 8 * (n - 64 * esc) + 16 * 64 * esc + runs
        assert bits / n == pytest.approx(escape_rows_cost(orc, w, lmax=lmax), rel=1e-12)


@pytest.mark.parametrize("shape,tile_cols,keep", [((9, 65), 64, 2), ((40, 300), 128, 4),
                                                   ((16, 1030), 512, 6), ((8, 256), 256, 1)])
def test_independent_reader_decodes_oracle_blobs(orc, shape, tile_cols, keep):
    """The pure-Python reader (tests/nwb1_reader.py), written from the format
    statement, reads the oracle's NWE1 blobs back to the input: the encoder is
    checked against the format, not only against the oracle's own decoder."""
    import nwb1_reader
    rng = np.random.default_rng(sum(shape) + keep)
    w = synth.to_bf16_bits(rng.standard_t(2, size=shape) * 0.02)
    blob = orc.escape_encode(w, tile_cols=tile_cols, lmax=7, keep=keep)
    h = nwb1_reader.parse(blob.tobytes())
    assert h["verbatim"] and h["kept"] == keep and h["verbatim_runs"] > 0
    assert np.array_equal(nwb1_reader.decode(blob.tobytes()), w)


def test_all_runs_escaped_closed_form(orc):
    """1.0 and 2.0 alternate, keep 1: every run holds 2.0, none is coded."""
    w = np.tile(np.array([0x3F80, 0x4000], dtype=np.uint16), (16, 512))   # 16 x 1024
    blob = orc.escape_encode(w, tile_cols=512, lmax=7, keep=1)
    tiles = 2 * 2
    chunk = 8 * 512 + 16 + 64 * 8 * 8 + 32
    assert blob.size == 512 + tiles * chunk
    assert _u64(blob, 96) == 0 and _u64(blob, 104) == tiles * 64 and not blob[128:384].any()
    assert (blob[512 + 4096:512 + 4096 + 8] == 0xFF).all()
    assert np.array_equal(orc.escape_decode(blob), w)


def test_every_pattern_round_trips(orc):
    allp = np.arange(65536, dtype=np.uint16).reshape(256, 256)
    for tile_cols in (64, 128, 256, 512):
        for keep, lmax in ((1, 7), (2, 7), (16, 7), (16, 12), (128, 7), (256, 12)):
            assert np.array_equal(orc.escape_decode(orc.escape_encode(allp, tile_cols, lmax, keep)),
                                  allp)
    rng = np.random.default_rng(4)
    shuffled = rng.permutation(allp.reshape(-1)).reshape(128, 512)
    assert np.array_equal(orc.escape_decode(orc.escape_encode(shuffled, keep=16, lmax=7)),
                          shuffled)
    for shape in ((1, 1), (1, 513), (9, 65), (77, 1030), (4100, 96)):
        w = synth.to_bf16_bits(rng.standard_t(3, size=shape) * 0.02)
        assert np.array_equal(orc.escape_decode(orc.escape_encode(w, tile_cols=128)), w)
    same = np.full((5, 70), 0xBF80, dtype=np.uint16)
    assert np.array_equal(orc.escape_decode(orc.escape_encode(same)), same)


def test_too_many_kept_symbols_for_the_limit_refused(orc):
    allp = np.arange(65536, dtype=np.uint16).reshape(256, 256)
    with pytest.raises(orc.OracleError):
        orc.escape_encode(allp, 512, 7, 256)       # 256 coded symbols cannot fit 7 bits


@pytest.mark.parametrize("name", synth.WORKLOADS)
def test_workload_generators_round_trip(orc, name):
    wl = synth.workload(name)
    for spec in wl.matrices[:2]:
        w = synth.matrix(spec, wl.seed, 0, min(spec.rows, 64)).reshape(-1, spec.cols)
        blob = orc.escape_encode(w)
        assert np.array_equal(orc.escape_decode(blob), w)
        # The 16 kept exponents cover nearly all weights: few runs escape.
        assert _u64(blob, 104) <= 0.25 * (w.size // 64)


def test_corrupt_blobs_refused(orc):
    exp = _golden("two_runs")
    w = _golden_matrix(exp)
    blob = orc.escape_encode(w, tile_cols=128, lmax=7, keep=1)
    fl = 512 + 1024
    run0_last = fl + 16 + 63

    def changed(off, val):
        b = blob.copy()
        b[off] = val
        return b

    cases = [changed(0, blob[0] ^ 1),               # magic
             changed(60, 0),                        # K = 0
             changed(104, 3),                       # escaped-run count
             changed(112, 1),                       # reserved header byte
             changed(fl, 0x06),                     # a flag for a group past the tile
             changed(fl + 8, 1),                    # flag padding
             changed(run0_last, 0x7F),              # an escaped run with only coded symbols
             changed(fl + 16 + 128, 3),             # a lane length: chunk size no longer adds up
             blob[:-16].copy()]                     # truncated
    for bad in cases:
        with pytest.raises(orc.OracleError) as e:
            orc.escape_decode(bad)
        assert e.value.code == CORRUPT
    # More coded symbols than kept ones.
    e2 = _golden("all_kept")
    b2 = orc.escape_encode(_golden_matrix(e2), tile_cols=64, lmax=7, keep=16)
    bad = b2.copy()
    bad[60] = 1
    with pytest.raises(orc.OracleError):
        orc.escape_decode(bad)


# ---- planted mistakes -------------------------------------------------------

MUTANTS = [
    ("kept ties to the larger symbol",
     "[&](int x, int y) { return cnt[x] > cnt[y]; });",
     "[&](int x, int y) { return cnt[x] > cnt[y] || (cnt[x] == cnt[y] && x > y); });"),
    ("rare test misses a run's last weight",
     "for (int c = 64 * m; c < 64 * m + 64; ++c) {\n          uint8_t s, rb;\n          tile_element(w, rows, cols, i, j, tile_rows, tile_cols, filler, g, c, &s, &rb);\n          if (!kept[s]) rare = true;",
     "for (int c = 64 * m; c < 64 * m + 63; ++c) {\n          uint8_t s, rb;\n          tile_element(w, rows, cols, i, j, tile_rows, tile_cols, filler, g, c, &s, &rb);\n          if (!kept[s]) rare = true;"),
    ("flag bits row-major", "flags[(size_t)g] |= (uint8_t)(1u << m);",
     "flags[(size_t)m] |= (uint8_t)(1u << g);"),
    ("escaped runs stored group-major",
     "    for (int g = 0; g < tile_rows; ++g) {\n      for (int m = 0; m < groups; ++m) {\n        if (!is_escaped(g, m)) continue;",
     "    for (int m = 0; m < groups; ++m) {\n      for (int g = 0; g < tile_rows; ++g) {\n        if (!is_escaped(g, m)) continue;"),
    ("run byte from the lane's offset only", "s = runs[64 * at + (c - 64 * (k / 16))];",
     "s = runs[64 * at + (k % 16)];"),
    ("escaped runs also coded", "        if (is_escaped(r, k / 16)) continue;\n", ""),
    ("code counts include escaped runs", "        if (rare) {\n          ++n_escaped;\n          continue;\n        }",
     "        if (rare) ++n_escaped;"),
]


def _escape_pins_pass(orc):
    try:
        for case in ("all_kept", "one_run", "two_runs", "tie_keep"):
            test_hand_derived_escape_blobs(orc, case)
        rng = np.random.default_rng(5)
        w = synth.to_bf16_bits(rng.standard_t(2, size=(40, 300)) * 0.02)
        for tile_cols in (64, 256):
            if not np.array_equal(orc.escape_decode(orc.escape_encode(w, tile_cols, 7, 4)), w):
                return False
        test_size_runs_and_code_bits_recomputed(orc, (40, 200), 64, 3, 7)
        return True
    except Exception:
        return False


def test_real_oracle_passes_escape_pins(orc):
    assert _escape_pins_pass(orc)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_escape_mistake_is_caught(orc, tmp_path, name, old, new):
    src = orc.source()
    assert src.count(old) == 1, name
    path = orc.compile_variant(src.replace(old, new), os.path.join(tmp_path, "mutant.so"))
    with orc.use_library(path):
        caught = not _escape_pins_pass(orc)
    assert caught, f"planted mistake not caught: {name}"
