"""Format variants the pages describe, costed on the synthetic workloads (bits
per weight, CPU only), so that the choice of code and byte split rests on
numbers:

* this library: exponent bits 14..7 coded with the optimal code limited to 12
  or to 7 bits (the default), sign and fraction raw ("Unweight", "Compressing
  BF16 Weights");
* the literal byte split: the high byte (sign and exponent bits 14..8) coded,
  the low byte (exponent bit 7 and fraction) raw ("NWC — Neural Weight
  Compression", "How it works > Byte planes");
* a frequency-ranked unary code of exponent bits 14..8 with the sign as a raw
  bit and an escape for rare values ("NWC", "How it works > Prefix code instead
  of rANS", format v9): rank r < R costs r + 1 bits, the escape R bits plus the
  7-bit field;
* verbatim escape rows ("Unweight", "Compressing BF16 Weights": a run of 64
  weights holding a rare exponent is stored whole): the 16 most frequent
  exponents get an optimal code (12-bit limit), a run of 64 consecutive weights
  of a matrix row that holds any other exponent costs 16 bits per weight, and
  every run carries a 1-bit flag.

`PYTHONPATH=. python tests/test_format_variants_cpu.py` prints the table."""
import numpy as np
import pytest

from lossless_bf16_weight_nwc_b200 import synth

NAMES = ["single_1024", "attn_4096_outliers", "mlp_pair_t5", "qwen3_4b_stack",
         "llama31_8b_stack"]


def _code_cost(orc, cnt, lmax):
    full = np.zeros(256, dtype=np.uint64)
    full[:cnt.size] = cnt
    lengths = orc.code_lengths(full, lmax).astype(np.float64)[:cnt.size]
    return float((cnt * lengths).sum() / cnt.sum())


def _entropy(cnt):
    q = cnt[cnt > 0] / cnt.sum()
    return float(-(q * np.log2(q)).sum())


def unary_rank_cost(cnt, ranks: int, literal_bits: int) -> float:
    """Mean bits of a unary code over the symbols ranked by frequency: rank
    r < ranks costs r + 1 bits; the rest cost `ranks` bits of escape prefix
    plus the literal."""
    p = np.sort(cnt[cnt > 0])[::-1].astype(np.float64) / cnt.sum()
    r = np.arange(p.size)
    return float((p * np.where(r < ranks, r + 1, ranks + literal_bits)).sum())


def escape_rows_cost(orc, w: np.ndarray, common: int = 16, run: int = 64, lmax: int = 12) -> float:
    """Bits per weight of the verbatim-escape-row layout (see the module text):
    runs of `run` weights along a row, the `common` most frequent exponents
    coded (limit lmax), any run holding another exponent stored as 16-bit words."""
    e = ((w.astype(np.int64) >> 7) & 0xFF)
    cnt = np.bincount(e.reshape(-1), minlength=256)
    keep = np.zeros(256, dtype=bool)
    keep[sorted(range(256), key=lambda v: (-cnt[v], v))[:common]] = True
    rows, cols = e.shape
    pad = (-cols) % run
    runs = np.pad(e, ((0, 0), (0, pad)), constant_values=int(np.argmax(cnt))).reshape(rows, -1, run)
    rare_run = (~keep[runs]).any(axis=2)
    coded = np.zeros(256, dtype=np.int64)
    for v in range(256):
        if keep[v]:
            coded[v] = int(np.count_nonzero(runs[~rare_run] == v))
    lengths = np.zeros(256)
    if coded.sum():
        full = np.zeros(256, dtype=np.uint64)
        full[:] = coded
        lengths = orc.code_lengths(full, lmax).astype(np.float64)
    code_bits = float((coded * lengths).sum()) + 8.0 * coded.sum()
    verbatim_bits = 16.0 * run * rare_run.sum()
    return (code_bits + verbatim_bits + rare_run.size) / (rows * (cols + pad))


def variant_costs(orc, name: str, rows: int = 2048) -> dict:
    wl = synth.workload(name)
    spec = wl.matrices[0]
    w = synth.matrix(spec, wl.seed, 0, min(spec.rows, rows)).reshape(-1).astype(np.int64)
    exp8 = np.bincount((w >> 7) & 0xFF, minlength=256)
    high = np.bincount(w >> 8, minlength=256)
    exp7 = np.bincount((w >> 8) & 0x7F, minlength=128)
    return {
        "entropy_exp8": _entropy(exp8),
        "this_lmax12": 8 + _code_cost(orc, exp8, 12),
        "this_lmax7": 8 + _code_cost(orc, exp8, 7),
        "literal_lmax12": 8 + _code_cost(orc, high, 12),
        "rank_unary_R15": 8 + 1 + unary_rank_cost(exp7, 15, 7),
        "rank_unary_R7": 8 + 1 + unary_rank_cost(exp7, 7, 7),
        "exp7_optimal": 8 + 1 + _code_cost(orc, exp7, 12),
        "escape_rows_top16": escape_rows_cost(orc, w.reshape(min(spec.rows, rows), spec.cols)),
        "escape_rows_top16_lmax7": escape_rows_cost(orc, w.reshape(min(spec.rows, rows), spec.cols),
                                                    lmax=7),
    }


def test_unary_rank_cost_closed_forms():
    # Geometric frequencies 1/2, 1/4, ... are exactly what a unary code fits.
    cnt = np.array([2 ** (10 - i) for i in range(10)] + [1], dtype=np.int64)
    p = cnt / cnt.sum()
    expected = float((p * (np.arange(cnt.size) + 1)).sum())
    assert unary_rank_cost(cnt, 64, 7) == pytest.approx(expected)
    # Symbol order does not matter; an escape costs ranks + literal bits.
    assert unary_rank_cost(cnt[::-1].copy(), 64, 7) == pytest.approx(expected)
    assert unary_rank_cost(np.array([3, 1]), 1, 7) == pytest.approx((3 * 1 + 1 * 8) / 4)


@pytest.mark.parametrize("name", NAMES)
def test_variant_costs(orc, name):
    c = variant_costs(orc, name)
    # Both byte splits land within 0.15 bit of each other, near 10.6-10.9 bits.
    assert abs(c["this_lmax12"] - c["literal_lmax12"]) < 0.15
    assert 10.5 < c["this_lmax12"] < 10.9
    # The 7-bit limit costs 0.05 to 0.3 bit per weight.
    assert 0.05 < c["this_lmax7"] - c["this_lmax12"] < 0.3
    # The ranked unary code is within 0.02 bit of the optimal code of the same
    # field (limited to 12 bits, which the unary code with 15 ranks is not), even
    # cut at 7 ranks: the 7-bit exponent field is close to geometric.
    assert c["rank_unary_R15"] <= c["rank_unary_R7"]
    assert abs(c["rank_unary_R15"] - c["exp7_optimal"]) < 0.005
    assert c["rank_unary_R7"] - c["exp7_optimal"] < 0.02
    # Escape rows: never below the complete optimal code of the same byte split;
    # with the default's 7-bit limit, within 0.11 bit of the default either way.
    assert c["escape_rows_top16"] >= c["this_lmax12"] - 1e-9
    assert c["escape_rows_top16"] <= c["escape_rows_top16_lmax7"]
    assert abs(c["escape_rows_top16_lmax7"] - c["this_lmax7"]) < 0.11


def test_escape_rows_closed_forms(orc):
    # One exponent only: a 1-bit code, the raw byte and one flag bit per run.
    w = np.full((2, 128), 0x3F80, dtype=np.uint16)
    assert escape_rows_cost(orc, w) == pytest.approx(8 + 1 + 1 / 64)
    # Row 0 starts with 16 other exponents (0x30..0x3f, once each) and row 1
    # holds 0xfe once.  The common 16 are 0x7f and 0x30..0x3e (ties go to the
    # smaller value), so 0x3f and 0xfe are rare: runs (0, 0..63) and
    # (1, 0..63) are verbatim, the other two runs hold only 0x7f (1-bit code).
    w2 = w.copy()
    w2[0, :16] = (np.arange(0x30, 0x40, dtype=np.uint16) << 7)
    w2[1, 5] = 0x7F00
    expected = (128 * (8 + 1) + 128 * 16 + 4) / 256
    assert escape_rows_cost(orc, w2) == pytest.approx(expected)


if __name__ == "__main__":
    import oracle
    keys = ["entropy_exp8", "this_lmax12", "this_lmax7", "literal_lmax12", "exp7_optimal",
            "rank_unary_R15", "rank_unary_R7", "escape_rows_top16", "escape_rows_top16_lmax7"]
    print("| workload | " + " | ".join(keys) + " |")
    print("|---" * (len(keys) + 1) + "|")
    for n in NAMES:
        c = variant_costs(oracle, n)
        print(f"| {n} | " + " | ".join(f"{c[k]:.3f}" for k in keys) + " |")
