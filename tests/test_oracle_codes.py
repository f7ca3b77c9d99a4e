"""Pins for the code-length (package-merge) and canonical-code steps of the oracle.

Independent checks: brute-force optimal length-limited codes on tiny alphabets,
Huffman's algorithm (heapq) where the limit does not bind, the Kraft equality,
the entropy bound, and the canonical-code worked examples of RFC 1951 §3.2.2.
"""
import heapq
import itertools
import math
import random

import numpy as np
import pytest

from conftest import golden_lines


def _cnt(weights, symbols=None):
    cnt = np.zeros(256, dtype=np.uint64)
    symbols = symbols or list(range(len(weights)))
    for s, w in zip(symbols, weights):
        cnt[s] = w
    return cnt


def _cost(cnt, lengths):
    return int(sum(int(c) * int(l) for c, l in zip(cnt, lengths)))


def _brute_force_cost(weights, lmax):
    best = None
    n = len(weights)
    for ls in itertools.product(range(1, lmax + 1), repeat=n):
        if sum(2.0 ** -l for l in ls) <= 1.0 + 1e-12:
            c = sum(w * l for w, l in zip(weights, ls))
            best = c if best is None else min(best, c)
    return best


def _huffman_lengths(weights):
    heap = [(w, i, (i,)) for i, w in enumerate(weights)]
    heapq.heapify(heap)
    depth = [0] * len(weights)
    uid = len(weights)
    while len(heap) > 1:
        w1, _, a = heapq.heappop(heap)
        w2, _, b = heapq.heappop(heap)
        for s in a + b:
            depth[s] += 1
        heapq.heappush(heap, (w1 + w2, uid, a + b))
        uid += 1
    return depth


def test_canonical_codes_rfc1951_examples(orc):
    rows = golden_lines("deflate_canonical_example.txt")
    for group in (rows[:8], rows[8:]):
        lengths = np.zeros(256, dtype=np.uint8)
        for sym, ln, _ in group:
            lengths[int(sym)] = int(ln)
        codes = orc.canonical_codes(lengths)
        for sym, ln, code in group:
            assert format(int(codes[int(sym)]), f"0{ln}b") == code


@pytest.mark.parametrize("n", [2, 3, 4, 5, 6, 7])
def test_package_merge_is_optimal_bruteforce(orc, n):
    rng = random.Random(n)
    for trial in range(12):
        weights = [rng.choice([1, 1, 2, 3, 5, 8, 13, 100, 1000]) for _ in range(n)]
        lo = max(1, math.ceil(math.log2(n)))
        for lmax in range(lo, min(n, 6) + 1):
            lengths = orc.code_lengths(_cnt(weights), lmax)
            got = [int(l) for l in lengths[:n]]
            assert max(got) <= lmax and min(got) >= 1
            assert abs(sum(2.0 ** -l for l in got) - 1.0) < 1e-12   # complete code
            assert sum(w * l for w, l in zip(weights, got)) == _brute_force_cost(weights, lmax)


def test_equals_huffman_when_limit_not_binding(orc):
    rng = np.random.default_rng(7)
    for trial in range(40):
        n = int(rng.integers(2, 60))
        weights = [int(v) for v in rng.integers(1, 10_000, size=n)]
        hl = _huffman_lengths(weights)
        syms = sorted(rng.choice(256, size=n, replace=False).tolist())
        lengths = orc.code_lengths(_cnt(weights, syms), 32)
        got = [int(lengths[s]) for s in syms]
        assert sum(w * l for w, l in zip(weights, got)) == sum(w * l for w, l in zip(weights, hl))
        if max(hl) <= 12:
            got12 = [int(orc.code_lengths(_cnt(weights, syms), 12)[s]) for s in syms]
            assert got12 == got


def test_limit_binds_on_fibonacci_weights(orc):
    fib = [1, 1]
    while len(fib) < 20:
        fib.append(fib[-1] + fib[-2])
    assert max(_huffman_lengths(fib)) == 19          # Huffman would go 19 deep
    for lmax in (5, 8, 12):
        lengths = orc.code_lengths(_cnt(fib), lmax)[:20]
        assert int(lengths.max()) == lmax
        assert abs(sum(2.0 ** -int(l) for l in lengths) - 1.0) < 1e-12
    # On a 7-symbol slice the limited code equals the brute-force optimum.
    small = fib[:7]
    for lmax in (3, 4, 5):
        got = orc.code_lengths(_cnt(small), lmax)[:7]
        assert sum(w * int(l) for w, l in zip(small, got)) == _brute_force_cost(small, lmax)


def test_entropy_bound(orc):
    rng = np.random.default_rng(3)
    for trial in range(20):
        n = int(rng.integers(2, 200))
        weights = rng.integers(1, 1 << 20, size=n).astype(np.float64)
        cnt = _cnt([int(w) for w in weights])
        lengths = orc.code_lengths(cnt, 32)[:n].astype(np.float64)
        p = weights / weights.sum()
        h = float(-(p * np.log2(p)).sum())
        avg = float((p * lengths).sum())
        assert h - 1e-9 <= avg < h + 1.0


def test_full_alphabet_and_edge_cases(orc):
    assert list(orc.code_lengths(np.ones(256, dtype=np.uint64), 8)) == [8] * 256
    with pytest.raises(orc.OracleError):
        orc.code_lengths(np.ones(256, dtype=np.uint64), 7)       # 256 > 2^7 codes
    one = np.zeros(256, dtype=np.uint64)
    one[77] = 5
    lengths = orc.code_lengths(one, 12)
    assert lengths[77] == 1 and lengths.sum() == 1


def test_canonical_codes_are_prefix_free(orc):
    rng = np.random.default_rng(11)
    for trial in range(20):
        cnt = np.zeros(256, dtype=np.uint64)
        syms = rng.choice(256, size=int(rng.integers(2, 256)), replace=False)
        cnt[syms] = rng.integers(1, 1 << 30, size=syms.size).astype(np.uint64)
        lengths = orc.code_lengths(cnt, 12)
        codes = orc.canonical_codes(lengths)
        words = [format(int(codes[s]), f"0{int(lengths[s])}b") for s in range(256) if lengths[s]]
        words.sort()
        for a, b in zip(words, words[1:]):
            assert not b.startswith(a)


def test_tie_rules_hand_derived(orc):
    for counts, lmax, expected in golden_lines("tie_break_cases.txt"):
        cnt = np.zeros(256, dtype=np.uint64)
        for item in counts.split(","):
            sym, c = item.split(":")
            cnt[int(sym)] = int(c)
        lengths = orc.code_lengths(cnt, int(lmax))
        for item in expected.split(","):
            sym, ln = item.split(":")
            assert int(lengths[int(sym)]) == int(ln), (counts, sym)


def test_filler_is_most_frequent_exponent(orc):
    import nwb1_reader
    # [2.5, 2.5, 1.5]: exponent 0x80 twice, 0x7f once -> filler 0x80
    blob = orc.encode(np.array([[0x4020, 0x4020, 0x3FC0]], dtype=np.uint16))
    assert nwb1_reader.parse(blob.tobytes())["filler"] == 0x80
