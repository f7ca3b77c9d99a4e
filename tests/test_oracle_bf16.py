"""Pins for the byte-plane split (oracle), against the Data Types page.

The split is checked two independent ways: against the page's worked examples
(tests/golden/bf16_worked_examples.txt) and, for all 65,536 patterns, against
what IEEE-style float arithmetic says the exponent and fraction fields are.
"""
import math

import numpy as np

from conftest import golden_lines
from lossless_bf16_weight_nwc_b200 import synth


def test_worked_examples(orc):
    for value, bits, s_hex, r_hex, _src in golden_lines("bf16_worked_examples.txt"):
        bits, s_exp, r_exp = int(bits, 16), int(s_hex, 16), int(r_hex, 16)
        if value not in ("nan", "+inf", "-inf", "+0", "-0", "+subnormal"):
            # numpy's own float32 -> bf16 rounding gives the page's bit pattern.
            assert int(synth.to_bf16_bits(np.array([float(value)]))[0]) == bits
        assert orc.plane_split(bits) == (s_exp, r_exp), value
        assert orc.plane_join(s_exp, r_exp) == bits


def test_split_matches_float_fields_all_patterns(orc):
    """For every pattern: s is the biased exponent and r = sign | fraction.

    Checked with float arithmetic only (no bit operations on the test side):
    s == 0 exactly for zeros/subnormals, s == 255 for inf/nan, otherwise
    2^(s-127) <= |v| < 2^(s-126) and (r & 0x7f) / 128 == |v| / 2^(s-127) - 1."""
    for bits in range(65536):
        s, r = orc.plane_split(bits)
        v = float(synth.bf16_bits_to_float(np.array([bits], dtype=np.uint16))[0])
        sign = 1 if math.copysign(1.0, v) < 0 else 0
        assert (r >> 7) == sign
        frac = r & 0x7F
        if math.isnan(v) or math.isinf(v):
            assert s == 255
            assert (frac == 0) == math.isinf(v)
        elif abs(v) < 2.0 ** -126:
            assert s == 0
            assert abs(v) == frac / 128.0 * 2.0 ** -126   # subnormal: fraction x 2^(1-bias)
        else:
            assert 2.0 ** (s - 127) <= abs(v) < 2.0 ** (s - 126)
            assert frac / 128.0 == abs(v) / 2.0 ** (s - 127) - 1.0
        assert orc.plane_join(s, r) == bits
