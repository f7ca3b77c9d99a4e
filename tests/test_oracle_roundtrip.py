"""Oracle round trip: decode(encode(W)) == W bit for bit ("Unweight" page:
bit-exact outputs; "NWC" page: decompressed weights bit-exact), over every BF16
pattern, odd shapes, every tile width and length limit, and degenerate inputs."""
import numpy as np
import pytest

from lossless_bf16_weight_nwc_b200 import synth

ALL = np.arange(65536, dtype=np.uint16)


@pytest.mark.parametrize("tile_cols,lmax", [(512, 12), (256, 10), (64, 8)])
def test_all_65536_patterns(orc, tile_cols, lmax):
    w = ALL.reshape(256, 256)
    assert np.array_equal(orc.decode(orc.encode(w, tile_cols=tile_cols, lmax=lmax)), w)


@pytest.mark.parametrize("shape", [(1, 65536), (65536, 1), (97, 677), (331, 199)])
def test_all_patterns_shuffled_odd_shapes(orc, shape):
    rng = np.random.default_rng(shape[0])
    flat = np.concatenate([rng.permutation(ALL), rng.permutation(ALL)])
    n = shape[0] * shape[1]
    w = flat[:n].reshape(shape)
    assert np.array_equal(orc.decode(orc.encode(w)), w)


@pytest.mark.parametrize("shape", [(1, 1), (8, 512), (7, 511), (9, 513), (16, 1025),
                                   (3, 64), (1, 4097)])
def test_config_generators_small_slices(orc, shape):
    for name in ("single_1024", "attn_4096_outliers", "mlp_pair_t5", "llama31_8b_stack"):
        wl = synth.workload(name)
        spec = wl.matrices[0]
        spec = synth.MatrixSpec(spec.name, shape[0], shape[1], spec.kind, spec.std, spec.tensor)
        w = synth.matrix(spec, wl.seed)
        for tile_cols in (512, 128):
            assert np.array_equal(orc.decode(orc.encode(w, tile_cols=tile_cols)), w)


def test_degenerate_inputs(orc):
    z = np.zeros((24, 600), dtype=np.uint16)                      # all +0
    assert np.array_equal(orc.decode(orc.encode(z)), z)
    one = np.full((5, 5), 0x3F80, dtype=np.uint16)                # single symbol 1.0
    assert np.array_equal(orc.decode(orc.encode(one)), one)
    # all 256 exponents present with equal counts -> every code is 8 bits
    w = (np.arange(256, dtype=np.uint16) << 7).reshape(1, 256).repeat(8, 0)
    blob = orc.encode(w, lmax=8)
    assert list(blob[128:384]) == [8] * 256
    assert np.array_equal(orc.decode(blob), w)
    specials = np.array([[0x0000, 0x8000, 0x0001, 0x807F, 0x7F80, 0xFF80, 0x7FC0, 0xFFFF]],
                        dtype=np.uint16)
    assert np.array_equal(orc.decode(orc.encode(specials)), specials)


def test_full_config1_matrix(orc):
    wl = synth.workload("single_1024")
    w = synth.matrix(wl.matrices[0], wl.seed)
    assert np.array_equal(orc.decode(orc.encode(w)), w)
