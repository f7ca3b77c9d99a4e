"""Statistics the pages state, checked on the synthetic inputs through the oracle.

* "Unweight" page, "Compressing BF16 Weights": the 16 most common exponents
  cover more than 99 % of a layer's weights.
* The coded exponent costs between its entropy H and H + 1 bits per weight (the
  length limit of 12 bits does not bind here), so Gaussian-init BF16 compresses
  by at least the 1.25x target: 16 bits -> 8 raw + ~2.6 coded + index."""
import numpy as np
import pytest

from lossless_bf16_weight_nwc_b200 import synth


@pytest.mark.parametrize("name", ["single_1024", "attn_4096_outliers", "mlp_pair_t5",
                                  "llama31_8b_stack"])
def test_exponent_concentration_and_ratio(orc, name):
    wl = synth.workload(name)
    spec = wl.matrices[0]
    rows = min(spec.rows, 1024)
    w = synth.matrix(spec, wl.seed, 0, rows)
    cnt = orc.histogram(w).astype(np.float64)
    p = np.sort(cnt / cnt.sum())[::-1]
    assert p[:16].sum() > 0.99
    q = cnt[cnt > 0] / cnt.sum()
    h = float(-(q * np.log2(q)).sum())
    lengths = orc.code_lengths(orc.histogram(w), 12).astype(np.float64)
    avg = float((cnt * lengths).sum() / cnt.sum())
    assert h <= avg < h + 1
    assert 2.3 < avg < 3.0
    blob = orc.encode(w)
    assert w.size * 2 / blob.size >= 1.25
