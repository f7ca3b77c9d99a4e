"""Property tests (hypothesis, CPU): for random shapes, tile widths, code
limits, rank counts, streams per lane and bit patterns -- NaN payloads, infinities, signed zeros
and subnormals included -- the library's host encoder writes exactly the
oracle's bytes for every code, the oracle decodes them back to the input, and
the library's size and schedule checks accept them."""
import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

SPECIAL = np.array([0x0000, 0x8000, 0x7F80, 0xFF80, 0x7FC0, 0xFFC1, 0x0001, 0x807F,
                    0x3F80, 0xBF80], dtype=np.uint16)


@pytest.fixture(scope="module")
def lib():
    from lossless_bf16_weight_nwc_b200 import build
    build.build()
    from lossless_bf16_weight_nwc_b200 import _lib
    return _lib


@st.composite
def matrices(draw):
    rows = draw(st.integers(1, 40))
    cols = draw(st.integers(1, 700))
    seed = draw(st.integers(0, 2**32 - 1))
    kind = draw(st.sampled_from(["normal", "wide", "bits", "special"]))
    rng = np.random.default_rng(seed)
    if kind == "normal":
        w = (rng.normal(0, 0.02, size=(rows, cols)).astype(np.float32).view(np.uint32) >> 16)
    elif kind == "wide":   # exponents over a wide range
        w = (rng.standard_cauchy(size=(rows, cols)).astype(np.float32).view(np.uint32) >> 16)
    elif kind == "bits":   # any pattern
        w = rng.integers(0, 65536, size=(rows, cols))
    else:                  # special values mixed into ordinary ones
        w = rng.choice(SPECIAL, size=(rows, cols))
    return np.ascontiguousarray(w.astype(np.uint16))


@settings(max_examples=200, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(w=matrices(), tile_cols=st.sampled_from([64, 128, 256, 512]),
       lmax=st.sampled_from([0, 8, 12]), threads=st.integers(1, 4),
       streams=st.sampled_from([1, 1, 2, 4]))
def test_prefix_code_matches_oracle(lib, orc, w, tile_cols, lmax, threads, streams):
    distinct = len(np.unique((w >> 7) & 0xFF))
    if lmax and (1 << lmax) < distinct:
        with pytest.raises(lib.NwcError):
            lib.nwc_plan(w, lmax=lmax, tile_cols=tile_cols, threads=threads)
        return
    plan = lib.nwc_plan(w, lmax=lmax, tile_cols=tile_cols, threads=threads, streams=streams)
    try:
        blob = lib.nwc_compress_host(plan, w)
        dev_bytes, _ = lib.nwc_plan_size(plan)
    finally:
        lib.nwc_plan_destroy(plan)
    used = int.from_bytes(blob[12:16].tobytes(), "little")
    assert np.array_equal(blob, orc.encode(w, tile_cols=tile_cols, lmax=used, streams=streams))
    assert np.array_equal(orc.decode(blob), w)
    if streams > 2:  # no kernel reads four streams per lane
        assert dev_bytes == 0
        return
    assert lib.nwc_blob_device_bytes(blob) == dev_bytes
    info, _, _, ring = lib.nwc_schedule_describe(blob)
    assert info["tiles"] == len(ring) == -(-w.shape[0] // 8) * -(-w.shape[1] // tile_cols)


@settings(max_examples=200, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(w=matrices(), tile_cols=st.sampled_from([64, 128, 256, 512]),
       ranks=st.integers(0, 7), threads=st.integers(1, 4))
def test_rank_code_matches_oracle(lib, orc, w, tile_cols, ranks, threads):
    plan = lib.nwc_plan(w, lmax=ranks, tile_cols=tile_cols, threads=threads,
                        code=lib.NWC_CODE_RANK)
    try:
        blob = lib.nwc_compress_host(plan, w)
    finally:
        lib.nwc_plan_destroy(plan)
    assert np.array_equal(blob, orc.rank_encode(w, tile_cols=tile_cols, ranks=ranks or 7))
    assert np.array_equal(orc.rank_decode(blob), w)


@settings(max_examples=150, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(w=matrices(), tile_cols=st.sampled_from([64, 128, 256, 512]),
       keep=st.sampled_from([1, 2, 5, 16, 64, 128, 256]), lmax=st.sampled_from([0, 5, 7]),
       threads=st.integers(1, 4))
def test_escape_code_matches_oracle(lib, orc, w, tile_cols, keep, lmax, threads):
    """The verbatim-run format (NWE1): the library's bytes are the oracle's, or
    both refuse (more coded exponents than lmax bits admit)."""
    try:
        ref = orc.escape_encode(w, tile_cols=tile_cols, lmax=lmax or 7, keep=keep)
    except orc.OracleError:
        with pytest.raises(lib.NwcError):
            lib.nwc_plan(w, lmax=lmax, tile_cols=tile_cols, threads=threads,
                         code=lib.NWC_CODE_ESCAPE, keep=keep)
        return
    plan = lib.nwc_plan(w, lmax=lmax, tile_cols=tile_cols, threads=threads,
                        code=lib.NWC_CODE_ESCAPE, keep=keep)
    try:
        blob = lib.nwc_compress_host(plan, w)
        dev_bytes, _ = lib.nwc_plan_size(plan)
    finally:
        lib.nwc_plan_destroy(plan)
    assert np.array_equal(blob, ref)
    assert np.array_equal(orc.escape_decode(blob), w)
    assert lib.nwc_blob_device_bytes(blob) == dev_bytes
