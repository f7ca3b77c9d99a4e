"""Property test of the launch schedule (hypothesis, CPU): for random matrices
(shape, tile width, code limit, value mix) and random devices (SM count,
shared-memory limit) and rows of x, every invariant the kernels rely on holds
(the checks of tests/test_schedule_cpu.py: exact bytes per copy, aligned
non-wrapping placement in the ring, releases awaited in order, bounded
outstanding copies, no overlap with any copy still outstanding), or the
library refuses the device as too small."""
import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from test_schedule_cpu import check_schedule


@pytest.fixture(scope="module")
def lib():
    from lossless_bf16_weight_nwc_b200 import build
    build.build()
    from lossless_bf16_weight_nwc_b200 import _lib
    return _lib


@st.composite
def blobs(draw):
    rows = draw(st.integers(1, 300))
    cols = draw(st.integers(1, 2100))
    tile_cols = draw(st.sampled_from([64, 128, 256, 512]))
    lmax = draw(st.sampled_from([0, 9, 12]))
    seed = draw(st.integers(0, 2**32 - 1))
    heavy = draw(st.booleans())
    rng = np.random.default_rng(seed)
    vals = rng.standard_cauchy((rows, cols)) * 0.01 if heavy else rng.normal(0, 0.02, (rows, cols))
    w = (vals.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    return w, tile_cols, lmax


@settings(max_examples=150, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(m=blobs(), sms=st.integers(1, 300), smem=st.integers(60_000, 232_448),
       rows_of_x=st.integers(0, 16))
def test_schedule_invariants_hold(lib, m, sms, smem, rows_of_x):
    w, tile_cols, lmax = m
    plan = lib.nwc_plan(w, lmax=lmax, tile_cols=tile_cols)
    blob = lib.nwc_compress_host(plan, w)
    lib.nwc_plan_destroy(plan)
    try:
        lib.nwc_schedule_describe(blob, sms, smem, rows_of_x)
    except lib.NwcError as e:
        assert e.status == 2                     # UNSUPPORTED: the device is too small
        return
    check_schedule(lib, blob, sms, smem, rows_of_x)
