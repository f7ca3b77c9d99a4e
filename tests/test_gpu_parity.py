"""GPU parity: the CUDA path (through the C ABI) against the oracle.

* Decompression must be bit-exact (integer/bit work): equal to the oracle's
  decode of the same matrix, for library-written and oracle-written blobs.
* GEMV must meet the tolerance of the target statement, per output
      |y_gpu - y_oracle| <= 1e-2 * ||W_n||_2 * ||x_b||_2 * 2^-8
  and overall ||y_gpu - y_oracle||_2 / ||y_oracle||_2 <= 2e-3,
  where y_oracle is the FP64 sum over the original BF16 weights.
"""
import numpy as np
import pytest

from lossless_bf16_weight_nwc_b200 import synth

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


def to_bf16(a: np.ndarray):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def bits(t) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def tolerance_check(y_gpu: np.ndarray, y_ref: np.ndarray, w: np.ndarray, x: np.ndarray):
    wf = synth.bf16_bits_to_float(w).astype(np.float64)
    xf = synth.bf16_bits_to_float(x).astype(np.float64)
    bound = 1e-2 * np.outer(np.linalg.norm(xf, axis=1), np.linalg.norm(wf, axis=1)) * 2.0 ** -8
    err = np.abs(y_gpu.astype(np.float64) - y_ref)
    worst = float((err / np.maximum(bound, 1e-300)).max())
    assert (err <= bound).all(), f"per-output bound exceeded: worst ratio {worst:.3g}"
    rel = np.linalg.norm(y_gpu - y_ref) / max(np.linalg.norm(y_ref), 1e-300)
    assert rel <= 2e-3, rel
    return worst, rel


def no_device_error(lib, *mats):
    """Each matrix's (or raw handle's) device error word is clear."""
    for m in mats:
        st, word = m.device_error() if hasattr(m, "device_error") else lib.nwc_get_device_error(m)
        assert st == 0, f"device error word {word:#x}"


SHAPES = [((8, 512), 512), ((9, 513), 512), ((77, 1030), 512), ((1, 2), 512),
          ((1000, 1026), 512), ((64, 4096), 512), ((129, 300), 256), ((40, 200), 128),
          ((17, 130), 64), ((4100, 96), 512)]


@pytest.mark.parametrize("lmax", [7, 12])
@pytest.mark.parametrize("shape,tile_cols", SHAPES)
def test_decompress_bit_exact(lib, orc, shape, tile_cols, lmax):
    spec = synth.MatrixSpec("w", shape[0], shape[1], "student_t5", 0.015, 1)
    w = synth.matrix(spec, 5)
    m = lib.CompressedMatrix.compress(w, tile_cols=tile_cols, lmax=lmax)
    out = bits(m.decompress())
    ref = orc.decode(orc.encode(w, tile_cols=tile_cols, lmax=lmax))
    assert np.array_equal(ref, w)
    assert np.array_equal(out, ref)
    no_device_error(lib, m)


def test_decompress_every_pattern(lib, orc):
    w = np.arange(65536, dtype=np.uint16).reshape(256, 256)
    for tile_cols, lmax in ((512, 12), (128, 8), (256, 0)):
        m = lib.CompressedMatrix.compress(w, tile_cols=tile_cols, lmax=lmax)
        assert np.array_equal(bits(m.decompress()), w)
        no_device_error(lib, m)
    rng = np.random.default_rng(0)
    shuffled = rng.permutation(w.reshape(-1)).reshape(128, 512)
    m = lib.CompressedMatrix.compress(shuffled)
    assert np.array_equal(bits(m.decompress()), shuffled)
    no_device_error(lib, m)


@pytest.mark.parametrize("lmax", [7, 9, 12])
def test_gpu_decodes_oracle_blob(lib, orc, lmax):
    spec = synth.MatrixSpec("w", 300, 2000, "normal_outliers", 1 / 64, 0)
    w = synth.matrix(spec, 1)
    blob = orc.encode(w, lmax=lmax)
    m = lib.CompressedMatrix.from_blob(blob)
    assert np.array_equal(bits(m.decompress()), w)
    x = synth.activations(1, 2, spec.cols)
    y = m.gemv(to_bf16(x)).cpu().numpy()
    tolerance_check(y, orc.gemv(w, x), w, x)
    no_device_error(lib, m)


@pytest.mark.parametrize("lmax", [0, 12])
@pytest.mark.parametrize("shape,tile_cols", SHAPES)
@pytest.mark.parametrize("batch", [1, 3, 8])
def test_gemv_parity_shapes(lib, orc, shape, tile_cols, batch, lmax):
    spec = synth.MatrixSpec("w", shape[0], shape[1], "normal", 0.02, 2)
    w = synth.matrix(spec, 6)
    x = synth.activations(6, batch, shape[1])
    m = lib.CompressedMatrix.compress(w, tile_cols=tile_cols, lmax=lmax)
    y = m.gemv(to_bf16(x)).cpu().numpy()
    tolerance_check(y, orc.gemv(w, x), w, x)
    no_device_error(lib, m)


@pytest.mark.parametrize("lmax", [0, 10])
@pytest.mark.parametrize("batch", [1, 2, 4, 5, 7, 8, 9, 16, 33, 64])
def test_gemv_every_batch(lib, orc, batch, lmax):
    spec = synth.MatrixSpec("w", 520, 2048, "normal_rowscale", 0.02, 3)
    w = synth.matrix(spec, 4)
    x = synth.activations(4, batch, spec.cols)
    m = lib.CompressedMatrix.compress(w, lmax=lmax)
    y = m.gemv(to_bf16(x)).cpu().numpy()
    tolerance_check(y, orc.gemv(w, x), w, x)
    no_device_error(lib, m)


def test_auto_lmax_and_fast_path(lib, orc):
    """Default plans use a 7-bit code limit (two codes per 14-bit peek) unless the
    matrix holds more than 128 distinct exponents."""
    w = synth.matrix(synth.MatrixSpec("w", 64, 1024, "normal", 0.02, 0), 3)
    plan = lib.nwc_plan(w)
    blob = lib.nwc_compress_host(plan, w)
    lib.nwc_plan_destroy(plan)
    assert int.from_bytes(blob[12:16].tobytes(), "little") == 7
    assert np.array_equal(blob, orc.encode(w, lmax=7))
    allp = np.arange(65536, dtype=np.uint16).reshape(128, 512)
    plan = lib.nwc_plan(allp)
    blob = lib.nwc_compress_host(plan, allp)
    lib.nwc_plan_destroy(plan)
    assert int.from_bytes(blob[12:16].tobytes(), "little") == 8


def test_gemv_deterministic_and_scratch_reuse(lib, orc):
    spec = synth.MatrixSpec("w", 2048, 4096, "normal", 0.02, 0)
    w = synth.matrix(spec, 8)
    x = synth.activations(8, 4, spec.cols)
    m = lib.CompressedMatrix.compress(w)
    xt = to_bf16(x)
    first = m.gemv(xt).cpu().numpy()
    for _ in range(20):
        again = m.gemv(xt).cpu().numpy()
        assert np.array_equal(first.view(np.uint32), again.view(np.uint32))
    tolerance_check(first, orc.gemv(w, x), w, x)
    no_device_error(lib, m)


@pytest.mark.parametrize("batch", [1, 16])
def test_fused_projections(lib, orc, batch):
    """q, k, v stacked into one matrix (one code table, one call): each part's
    slice of y meets the tolerance against that part alone."""
    parts = [synth.MatrixSpec(f"layers.0.{n}", r, 1536, "normal", 0.02, t)
             for t, (n, r) in enumerate((("q", 512), ("k", 128), ("v", 128)))]
    ws = [synth.matrix(p, 9) for p in parts]
    m = lib.CompressedMatrix.compress_fused(ws)
    assert m.row_splits == [0, 512, 640, 768] and m.rows == 768
    assert np.array_equal(bits(m.decompress()), np.concatenate(ws))
    x = synth.activations(9, batch, 1536)
    ys = m.split(m.gemv(to_bf16(x)))
    for w, y in zip(ws, ys):
        tolerance_check(y.cpu().numpy(), orc.gemv(w, x), w, x)
    no_device_error(lib, m)


def test_autotune_picks_a_timed_candidate(lib, orc):
    """The strategy autotuner times real candidates on the device (two formats,
    both kernels); the strategy it picks, applied, meets the tolerance."""
    from lossless_bf16_weight_nwc_b200 import autotune
    from lossless_bf16_weight_nwc_b200.autotune import Strategy
    spec = synth.MatrixSpec("w", 1024, 4096, "normal", 0.02, 0)
    w = synth.matrix(spec, 3)
    cands = [Strategy(512, 0, 1, "prefix", "cuda"), Strategy(512, 0, 1, "prefix", "tensor"),
             Strategy(256, 0, 2, "prefix", "cuda"), Strategy(512, 0, 1, "rank", "tensor")]
    choice = autotune.Tuner().tune(w, 16, candidates=cands, reps=5)
    assert choice.strategy in cands
    assert set(choice.timings) == {c.key for c in cands} and min(choice.timings.values()) > 0
    s = choice.strategy
    m = lib.CompressedMatrix.compress(w, tile_cols=s.tile_cols, lmax=s.lmax, streams=s.streams,
                                      code=lib.NWC_CODE_RANK if s.code == "rank" else 0)
    autotune.apply(m, s)
    x = synth.activations(3, 16, spec.cols)
    xt = to_bf16(x)
    assert lib.nwc_gemv_path(m.handle, xt, 16)[1] == (s.kernel == "tensor")
    tolerance_check(m.gemv(xt).cpu().numpy(), orc.gemv(w, x), w, x)
    no_device_error(lib, m)


def test_sharded_matrix_single_process(lib, orc):
    """A row-sharded matrix in one process (world 1, no collective) runs the
    library on its one shard and meets the tolerance."""
    from lossless_bf16_weight_nwc_b200 import sharded
    spec = synth.MatrixSpec("w", 300, 1024, "normal", 0.02, 0)
    w = synth.matrix(spec, 7)
    m = sharded.ShardedMatrix.compress(w)
    assert m.ranges == [(0, 300)] and m.local is not None
    x = synth.activations(7, 2, spec.cols)
    tolerance_check(m.gemv(to_bf16(x)).cpu().numpy(), orc.gemv(w, x), w, x)
    no_device_error(lib, m.local)
    m.close()


@pytest.mark.parametrize("batch", [1, 2, 5, 16, 40])
@pytest.mark.parametrize("cols", [1, 3, 513, 1025, 4097])
def test_gemv_odd_columns(lib, orc, cols, batch):
    """An odd number of columns: x rows start on 2-byte boundaries, read one
    element at a time; staged in shared memory or read directly."""
    spec = synth.MatrixSpec("w", 300, cols, "normal", 0.02, 1)
    w = synth.matrix(spec, 3)
    x = synth.activations(3, batch, cols)
    m = lib.CompressedMatrix.compress(w)
    xt = to_bf16(x)
    assert lib.nwc_gemv_path(m.handle, xt, batch)[1] is False
    tolerance_check(m.gemv(xt).cpu().numpy(), orc.gemv(w, x), w, x)
    no_device_error(lib, m)


def test_gemv_into_pinned_host_memory(lib, orc):
    """y may be pinned host memory the device can address: the kernel stores the
    result there directly."""
    spec = synth.MatrixSpec("w", 1000, 2048, "normal", 0.02, 0)
    w = synth.matrix(spec, 5)
    x = synth.activations(5, 3, spec.cols)
    m = lib.CompressedMatrix.compress(w)
    yh = torch.full((3, spec.rows), float("nan"), dtype=torch.float32).pin_memory()
    lib.nwc_gemv(m.handle, to_bf16(x), yh, 3)
    torch.cuda.synchronize()
    tolerance_check(yh.numpy(), orc.gemv(w, x), w, x)
    no_device_error(lib, m)


@pytest.mark.parametrize("lmax", [0, 12])
@pytest.mark.parametrize("shape,tile_cols", [((77, 1030), 256), ((1000, 2048), 512), ((9, 64), 64),
                                             ((4100, 96), 512)])
def test_gather_rows(lib, shape, tile_cols, lmax):
    """Embedding lookup from the compressed matrix: bit-exact rows."""
    spec = synth.MatrixSpec("w", shape[0], shape[1], "student_t5", 0.015, 2)
    w = synth.matrix(spec, 8)
    m = lib.CompressedMatrix.compress(w, tile_cols=tile_cols, lmax=lmax)
    rng = np.random.default_rng(3)
    ids = np.concatenate([[0, shape[0] - 1], rng.integers(0, shape[0], 37)]).astype(np.int32)
    out = m.gather_rows(torch.from_numpy(ids).cuda())
    assert np.array_equal(bits(out), w[ids])
    no_device_error(lib, m)


def test_gather_rows_every_pattern(lib):
    """All 65,536 BF16 patterns (NaN payloads, infinities, zeros), which need
    lmax 8 and the 12-bit table."""
    w = np.arange(65536, dtype=np.uint16).reshape(256, 256)
    m = lib.CompressedMatrix.compress(w)
    ids = np.arange(255, -1, -1, dtype=np.int32)
    assert np.array_equal(bits(m.gather_rows(torch.from_numpy(ids).cuda())), w[ids])
    no_device_error(lib, m)


def test_gather_rows_out_of_range(lib):
    w = synth.matrix(synth.MatrixSpec("w", 24, 512, "normal", 0.02, 0), 1)
    m = lib.CompressedMatrix.compress(w)
    out = torch.zeros((2, 512), dtype=torch.int16, device="cuda")
    ids = torch.tensor([5, 24], dtype=torch.int32, device="cuda")
    lib.nwc_gather_rows(m.handle, ids, 2, out)
    st, word = m.device_error()
    assert st == 1 and word & 4                     # INVALID_ARG: a row id out of range
    assert np.array_equal(out[0].cpu().numpy().view(np.uint16), w[5])
    assert not out[1].any()                         # left unwritten
    no_device_error(lib, m)


def test_handle_from_device_image(lib, orc):
    spec = synth.MatrixSpec("w", 96, 1536, "normal", 0.02, 0)
    w = synth.matrix(spec, 2)
    m = lib.CompressedMatrix.compress(w)
    copy = m.image.clone()
    h = lib.nwc_handle_from_device(copy, copy.numel())
    out = torch.empty((96, 1536), dtype=torch.bfloat16, device="cuda")
    lib.nwc_decompress(h, out)
    assert np.array_equal(bits(out), w)
    no_device_error(lib, h, m)
    lib.nwc_handle_destroy(h)


def test_invalid_arguments_rejected(lib):
    w = synth.matrix(synth.MatrixSpec("w", 16, 1024, "normal", 0.02, 0), 0)
    m = lib.CompressedMatrix.compress(w)
    x = torch.zeros((1, 1024), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((1, 16), dtype=torch.float32, device="cuda")
    with pytest.raises(lib.NwcError):
        lib.nwc_gemv(m.handle, x, y, 0)
    with pytest.raises(lib.NwcError):
        lib.nwc_gemv(m.handle, x, y, 65)
    with pytest.raises(lib.NwcError):            # misaligned x
        lib.nwc_gemv(m.handle, x.data_ptr() + 2, y, 1)
    odd = lib.CompressedMatrix.compress(synth.matrix(synth.MatrixSpec("w", 4, 5, "normal", 0.02, 0), 0))
    x5 = torch.zeros((2, 5), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.NwcError):            # x of an odd-width matrix on an odd address
        lib.nwc_gemv(odd.handle, x5.data_ptr() + 1, torch.zeros(4, device="cuda"), 1)
    blob = np.zeros(1024, dtype=np.uint8)
    with pytest.raises(lib.NwcError):
        lib.CompressedMatrix.from_blob(blob)
    with pytest.raises(ValueError):              # x in host memory never reaches a kernel
        m.gemv(torch.zeros((1, 1024), dtype=torch.bfloat16))
    with pytest.raises(ValueError):              # nor a y smaller than the output
        m.gemv(x, y=torch.zeros((1, 15), dtype=torch.float32, device="cuda"))
    assert m.gather_rows(torch.tensor([3, 0])).shape == (2, 1024)  # host ids are moved
    no_device_error(lib, m)


# ---- the benchmark workloads at full size ------------------------------------

@pytest.mark.parametrize("name", ["single_1024", "attn_4096_outliers"])
def test_workload_full_parity(lib, orc, name):
    wl = synth.workload(name)
    for spec in wl.matrices:
        w = synth.matrix(spec, wl.seed)
        m = lib.CompressedMatrix.compress(w)
        assert np.array_equal(bits(m.decompress()), w)
        assert m.ratio >= 1.25
        for batch in wl.batches:
            x = synth.activations(wl.seed, batch, spec.cols)
            y = m.gemv(to_bf16(x)).cpu().numpy()
            tolerance_check(y, orc.gemv(w, x), w, x)
        no_device_error(lib, m)
        m.close()


def test_workload_mlp_pair_full(lib, orc):
    wl = synth.workload("mlp_pair_t5")
    for spec in wl.matrices:
        w = synth.matrix(spec, wl.seed)
        m = lib.CompressedMatrix.compress(w)
        assert np.array_equal(bits(m.decompress()), w)
        for batch in wl.batches:
            x = synth.activations(wl.seed, batch, spec.cols)
            y = m.gemv(to_bf16(x)).cpu().numpy()
            tolerance_check(y, orc.gemv(w, x), w, x)
        no_device_error(lib, m)
        m.close()
