"""GPU parity at the full sizes of the two layer stacks (Qwen3-4B- and
Llama-3.1-8B-shaped): every distinct matrix shape of a layer, plus the
lm_head, compressed through the C ABI, decompressed bit-exact (checked on the
device against the original), and multiplied at the stack's batch sizes.  y
is compared with the oracle's FP64 sum on 256 sampled rows of each matrix
(first and last row included), with the tolerance of tests/test_gpu_parity.py.
The lm_head is its first rows repeated (synth.head_matrix), at full shape.
The stacked projections the per-token benchmark runs with --fuse (qkv,
gate_up) are checked the same way, part by part."""
import numpy as np
import pytest

from lossless_bf16_weight_nwc_b200 import synth
from test_gpu_parity import no_device_error, tolerance_check, to_bf16

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


@pytest.mark.parametrize("name", ["qwen3_4b_stack", "llama31_8b_stack"])
def test_stack_shapes_full_size(lib, orc, name):
    wl, layer0, head, _ = synth.stack_parts(name)
    for spec in layer0 + [head]:
        w = synth.head_matrix(spec, wl.seed) if spec is head else synth.matrix(spec, wl.seed)
        m = lib.CompressedMatrix.compress(w)
        assert m.ratio >= 1.25, (spec.name, m.ratio)
        original = torch.from_numpy(w.view(np.int16)).cuda()
        out = m.decompress()
        assert torch.equal(out.view(torch.int16), original), spec.name
        del out, original
        idx = np.unique(np.linspace(0, spec.rows - 1, 256).astype(np.int64))
        for batch in wl.batches:
            x = synth.activations(wl.seed, batch, spec.cols)
            y = m.gemv(to_bf16(x)).cpu().numpy()
            tolerance_check(y[:, idx], orc.gemv(w[idx], x), w[idx], x)
        no_device_error(lib, m)
        m.close()


@pytest.mark.parametrize("name", ["qwen3_4b_stack", "llama31_8b_stack"])
def test_stacked_projections_full_size(lib, orc, name):
    wl, layer0, _, _ = synth.stack_parts(name)
    for group, parts in synth.fused_layer(layer0):
        if len(parts) == 1:
            continue
        ws = [synth.matrix(p, wl.seed) for p in parts]
        m = lib.CompressedMatrix.compress_fused(ws)
        assert m.ratio >= 1.25, (group, m.ratio)
        for batch in wl.batches:
            x = synth.activations(wl.seed, batch, parts[0].cols)
            ys = m.split(m.gemv(to_bf16(x)))
            for p, w, y in zip(parts, ws, ys):
                idx = np.unique(np.linspace(0, p.rows - 1, 128).astype(np.int64))
                tolerance_check(y.cpu().numpy()[:, idx], orc.gemv(w[idx], x), w[idx], x)
        no_device_error(lib, m)
        m.close()
