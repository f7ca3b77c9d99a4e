"""GPU parity of the tensor-core (tcgen05) GEMV kernel against the FP64 oracle.

The kernel decodes each tile once into shared memory and multiplies it with
every row of x on the tensor cores ("Unweight", "Direct GPU Decompression").
Its CTAs own rectangles of tiles (a row range x a column range; K is split
into several column ranges when a CTA would otherwise own too few rows to
keep its decode warps busy, and the parts' sums meet in scratch slots), so
these shapes cover: a single column tile, many column tiles, a K split in two
and in four with ragged row ranges, fewer row tiles than SMs, ragged rows and
columns (a partial last 64-column chunk read by TMA past the end of x), every
tile width, both code limits, and every accumulator width (16, 32, 64
columns).

The tolerance is the parity tests' (per output and overall L2) against the
oracle's FP64 GEMV over the original BF16 weights.
"""
import numpy as np
import pytest

from lossless_bf16_weight_nwc_b200 import synth
from test_gpu_parity import no_device_error, to_bf16, tolerance_check

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from lossless_bf16_weight_nwc_b200 import build
    build.build()
    from lossless_bf16_weight_nwc_b200 import _lib
    torch.cuda.set_device(0)
    return _lib


def tc_gemv(lib, m, x):
    """y through nwc_gemv with the tensor-core kernel forced at any batch."""
    lib.nwc_gemv_set_tc_min_batch(m.handle, 1)
    xt = to_bf16(x)
    launches, tc = lib.nwc_gemv_path(m.handle, xt, x.shape[0])
    assert tc and launches == 1
    y = torch.full((x.shape[0], m.rows), float("nan"), dtype=torch.float32, device="cuda")
    lib.nwc_gemv(m.handle, xt, y, x.shape[0])
    torch.cuda.synchronize()
    return y.cpu().numpy()


SHAPES = [((8, 512), 512), ((300, 2000), 512), ((1024, 1024), 512), ((77, 1032), 512),
          ((129, 296), 256), ((40, 200), 128), ((17, 136), 64), ((4100, 96), 512),
          ((2048, 4096), 512), ((520, 14336), 512), ((96, 512), 512), ((1000, 8192), 512)]


@pytest.mark.parametrize("lmax", [0, 12])
@pytest.mark.parametrize("shape,tile_cols", SHAPES)
@pytest.mark.parametrize("batch", [1, 16, 33, 64])
def test_tc_parity_shapes(lib, orc, shape, tile_cols, batch, lmax):
    spec = synth.MatrixSpec("w", shape[0], shape[1], "normal_outliers", 1 / 64, 3)
    w = synth.matrix(spec, 21)
    x = synth.activations(21, batch, spec.cols)
    m = lib.CompressedMatrix.compress(w, tile_cols=tile_cols, lmax=lmax)
    tolerance_check(tc_gemv(lib, m, x), orc.gemv(w, x), w, x)
    no_device_error(lib, m)


@pytest.mark.parametrize("batch", list(range(1, 65, 7)) + [16, 17, 32, 48, 63, 64])
def test_tc_every_width(lib, orc, batch):
    spec = synth.MatrixSpec("w", 1000, 3072, "student_t5", 0.015, 1)
    w = synth.matrix(spec, 4)
    x = synth.activations(4, batch, spec.cols)
    m = lib.CompressedMatrix.compress(w)
    tolerance_check(tc_gemv(lib, m, x), orc.gemv(w, x), w, x)
    no_device_error(lib, m)


def test_tc_deterministic_and_default_threshold(lib, orc):
    """Reruns give the same bits; batches of 17 and more take the tensor-core
    kernel by default, up to 16 the CUDA-core kernel (one launch), and both
    meet the tolerance."""
    spec = synth.MatrixSpec("w", 2048, 4096, "normal", 0.02, 0)
    w = synth.matrix(spec, 8)
    m = lib.CompressedMatrix.compress(w)
    for batch, want_tc in ((8, False), (16, False), (17, True), (40, True)):
        x = synth.activations(8, batch, spec.cols)
        xt = to_bf16(x)
        launches, tc = lib.nwc_gemv_path(m.handle, xt, batch)
        assert tc == want_tc and launches == 1
        first = m.gemv(xt).cpu().numpy()
        for _ in range(5):
            assert np.array_equal(first.view(np.uint32), m.gemv(xt).cpu().numpy().view(np.uint32))
        tolerance_check(first, orc.gemv(w, x), w, x)
    lib.nwc_gemv_set_tc_min_batch(m.handle, 0)        # never: 64 rows in 4 launches
    assert lib.nwc_gemv_path(m.handle, to_bf16(synth.activations(8, 64, spec.cols)), 64) == (4, False)
    no_device_error(lib, m)


def test_tc_unaligned_x_takes_cuda_cores(lib, orc):
    """x not 16-byte aligned cannot be read by TMA: the CUDA-core kernel runs."""
    spec = synth.MatrixSpec("w", 256, 1024, "normal", 0.02, 0)
    w = synth.matrix(spec, 2)
    x = synth.activations(2, 20, spec.cols)
    m = lib.CompressedMatrix.compress(w)
    buf = torch.zeros(20 * 1024 + 2, dtype=torch.bfloat16, device="cuda")
    xt = buf[2:].view(20, 1024)
    xt.copy_(to_bf16(x))
    assert lib.nwc_gemv_path(m.handle, xt, 20) == (2, False)
    y = torch.empty((20, 256), dtype=torch.float32, device="cuda")
    lib.nwc_gemv(m.handle, xt, y, 20)
    tolerance_check(y.cpu().numpy(), orc.gemv(w, x), w, x)
    no_device_error(lib, m)


@pytest.mark.parametrize("batch", [16, 33, 64])
def test_tc_llama_shapes_full_size(lib, orc, batch):
    """Every distinct matrix shape of the Llama-3.1-8B-shaped stack at full
    size (the lm_head 128256 x 4096 included), sampled rows against the oracle."""
    wl, layer0, head, _ = synth.stack_parts("llama31_8b_stack")
    seen = set()
    for spec in layer0 + [head]:
        if (spec.rows, spec.cols) in seen:
            continue
        seen.add((spec.rows, spec.cols))
        w = synth.head_matrix(spec, wl.seed) if spec is head else synth.matrix(spec, wl.seed)
        m = lib.CompressedMatrix.compress(w)
        lib.nwc_gemv_set_tc_min_batch(m.handle, 1)
        x = synth.activations(wl.seed, batch, spec.cols)
        xt = to_bf16(x)
        assert lib.nwc_gemv_path(m.handle, xt, batch) == (1, True)
        y = m.gemv(xt).cpu().numpy()
        idx = np.unique(np.concatenate([np.linspace(0, spec.rows - 1, 256).astype(np.int64),
                                        np.arange(0, 64), np.arange(spec.rows - 64, spec.rows)]))
        tolerance_check(y[:, idx], orc.gemv(w[idx], x), w[idx], x)
        no_device_error(lib, m)
        m.close()
