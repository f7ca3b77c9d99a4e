"""The pins must catch plausible mistakes: each case below plants one mistake in
a copy of the oracle source (on the CPU), builds it, and checks that at least
one pin fails.  The real oracle is never modified."""
import os

import numpy as np
import pytest

import nwb1_reader
from conftest import golden_lines
from lossless_bf16_weight_nwc_b200 import synth

# (name, original text, planted text); every original must occur exactly once.
MUTANTS = [
    ("exponent field shifted", "*s = (uint8_t)((w >> 7) & 0xFF);", "*s = (uint8_t)((w >> 8) & 0xFF);"),
    ("sign bit dropped on join", "((uint16_t)(r >> 7) << 15)", "((uint16_t)(r >> 7) << 14)"),
    ("one item too many selected", "for (size_t q = 0; q < 2 * n - 2; ++q)",
     "for (size_t q = 0; q < 2 * n - 1; ++q)"),
    ("canonical step loses a bit", "next = (next + 1) << (l - prev_len);",
     "next = (next + 1) << (l > prev_len ? l - prev_len - 1 : 0);"),
    ("lane owns strided columns", "*c = 64 * (k / 16) + 16 * (t % 4) + (k % 16);",
     "*c = 64 * (k / 16) + 4 * (k % 16) + (t % 4);"),
    ("lane row from the wrong bits", "*r = t / 4;", "*r = t % 8;"),
    ("raw plane lane-major", "int raw_position(int t, int k) { return (k / 16) * 512 + 16 * t + (k % 16); }",
     "int raw_position(int t, int k) { return (k / 16) * 512 + t + 32 * (k % 16); }"),
    ("filler is least frequent", "if (cnt[s] > cnt[best]) best = s;",
     "if (cnt[s] && (cnt[best] == 0 || cnt[s] < cnt[best])) best = s;"),
    ("histogram skips last weight", "for (int64_t n = 0; n < rows * cols; ++n) {",
     "for (int64_t n = 0; n + 1 < rows * cols; ++n) {"),
    ("gemv drops a term", "for (int64_t k = 0; k < cols; ++k)\n        acc +=",
     "for (int64_t k = 1; k < cols; ++k)\n        acc +="),
    ("gemv transposed operand", "bf16_to_double(w[n * cols + k])", "bf16_to_double(w[k * rows % (rows * cols) + n])"),
    ("leaf weight ties reversed", "return a.symbol < b.symbol;", "return a.symbol > b.symbol;"),
]


def _pins_pass(orc):
    """A compact run of the pins; returns False at the first failing one."""
    try:
        for value, bits, s_hex, r_hex, _ in golden_lines("bf16_worked_examples.txt"):
            if orc.plane_split(int(bits, 16)) != (int(s_hex, 16), int(r_hex, 16)):
                return False
            if orc.plane_join(int(s_hex, 16), int(r_hex, 16)) != int(bits, 16):
                return False
        rows = golden_lines("deflate_canonical_example.txt")[:8]
        lengths = np.zeros(256, dtype=np.uint8)
        for sym, ln, _ in rows:
            lengths[int(sym)] = int(ln)
        codes = orc.canonical_codes(lengths)
        if any(format(int(codes[int(s)]), f"0{l}b") != c for s, l, c in rows):
            return False
        cnt = np.zeros(256, dtype=np.uint64)
        cnt[:5] = [1, 1, 2, 3, 5]
        if orc.code_lengths(cnt, 12)[:5].tolist() != [4, 4, 3, 2, 1]:
            return False
        w2 = np.array([[0x4020, 0x3FC0]], dtype=np.uint16)
        b2 = orc.encode(w2)
        if b2[512 + 1] != 0x40 or int(orc.blob_info(b2)[1]) != 2:
            return False
        if bytes(b2[56:57]) != b"\x7f":                   # filler symbol (tie)
            return False
        b3 = orc.encode(np.array([[0x4020, 0x4020, 0x3FC0]], dtype=np.uint16))
        if bytes(b3[56:57]) != b"\x80":                   # filler symbol (majority)
            return False
        for counts, lmax, expected in golden_lines("tie_break_cases.txt"):
            cnt = np.zeros(256, dtype=np.uint64)
            for item in counts.split(","):
                cnt[int(item.split(":")[0])] = int(item.split(":")[1])
            got = orc.code_lengths(cnt, int(lmax))
            if any(int(got[int(e.split(":")[0])]) != int(e.split(":")[1])
                   for e in expected.split(",")):
                return False
        rng = np.random.default_rng(5)
        w = synth.to_bf16_bits(rng.normal(0, 0.02, size=(9, 600)))
        blob = orc.encode(w)
        if not np.array_equal(orc.decode(blob), w):
            return False
        if not np.array_equal(nwb1_reader.decode(blob.tobytes()), w):
            return False
        h = nwb1_reader.parse(blob.tobytes())
        if sum(orc.histogram(w)) != w.size:
            return False
        x = synth.to_bf16_bits(rng.normal(0, 1, size=(1, 600)))
        y = orc.gemv(w, x)
        wf = synth.bf16_bits_to_float(w).astype(np.float64)
        xf = synth.bf16_bits_to_float(x).astype(np.float64)
        if np.abs(y - xf @ wf.T).max() > 1e-9:
            return False
        return h["coded_bits"] > 0
    except Exception:
        return False


def test_real_oracle_passes_compact_pins(orc):
    assert _pins_pass(orc)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(orc, tmp_path, name, old, new):
    src = orc.source()
    assert src.count(old) == 1, name
    path = orc.compile_variant(src.replace(old, new), os.path.join(tmp_path, "mutant.so"))
    with orc.use_library(path):
        caught = not _pins_pass(orc)
    assert caught, f"planted mistake not caught: {name}"
