"""Pins for the oracle's FP64 matrix-vector product over the original BF16 W.

y[b][n] = sum_k W[n][k] x[b][k].  Checked against exact integer arithmetic,
one-hot selection, and Python's exactly rounded math.fsum (each BF16 x BF16
product is exact in FP64, so fsum gives the correctly rounded sum)."""
import math

import numpy as np

from lossless_bf16_weight_nwc_b200 import synth


def _f(bits):
    return synth.bf16_bits_to_float(bits).astype(np.float64)


def test_integer_valued_exact(orc):
    rng = np.random.default_rng(0)
    for trial in range(20):
        n, k, b = (int(v) for v in rng.integers(1, 9, size=3))
        wi = rng.integers(-64, 65, size=(n, k))
        xi = rng.integers(-64, 65, size=(b, k))
        w = synth.to_bf16_bits(wi.astype(np.float64))
        x = synth.to_bf16_bits(xi.astype(np.float64))
        y = orc.gemv(w, x)
        exact = [[sum(int(wi[r, c]) * int(xi[bb, c]) for c in range(k)) for r in range(n)]
                 for bb in range(b)]
        assert np.array_equal(y, np.array(exact, dtype=np.float64))


def test_one_hot_selects_columns(orc):
    rng = np.random.default_rng(1)
    w = synth.to_bf16_bits(rng.normal(0, 0.02, size=(33, 70)))
    for c in (0, 17, 69):
        x = np.zeros((1, 70), dtype=np.uint16)
        x[0, c] = 0x3F80                                   # 1.0
        assert np.array_equal(orc.gemv(w, x)[0], _f(w[:, c]))
        x[0, c] = 0xC000                                   # -2.0
        assert np.array_equal(orc.gemv(w, x)[0], -2.0 * _f(w[:, c]))


def test_matches_exactly_rounded_sum(orc):
    rng = np.random.default_rng(2)
    for trial in range(10):
        n, k, b = int(rng.integers(1, 20)), int(rng.integers(1, 3000)), int(rng.integers(1, 4))
        w = synth.to_bf16_bits(rng.normal(0, 0.02, size=(n, k)))
        x = synth.to_bf16_bits(rng.normal(0, 1, size=(b, k)))
        y = orc.gemv(w, x)
        wf, xf = _f(w), _f(x)
        for bb in range(b):
            for r in range(n):
                terms = wf[r] * xf[bb]                     # exact products
                ref = math.fsum(terms)
                bound = k * 2.0 ** -52 * float(np.abs(terms).sum())
                assert abs(y[bb, r] - ref) <= bound


def test_row_range(orc):
    rng = np.random.default_rng(3)
    w = synth.to_bf16_bits(rng.normal(0, 0.02, size=(40, 90)))
    x = synth.to_bf16_bits(rng.normal(0, 1, size=(2, 90)))
    full = orc.gemv(w, x)
    part = orc.gemv(w, x, 10, 25)
    assert np.array_equal(part[:, 10:25], full[:, 10:25])
    assert not part[:, :10].any() and not part[:, 25:].any()
