"""Fused projections on the CPU: which matrices of a layer are stacked, that
the stacked matrix is the parts' rows in order, that the oracle's result for the
stacked matrix is the parts' results side by side, and the binding's checks and
output split (no GPU calls)."""
import numpy as np
import pytest

from lossless_bf16_weight_nwc_b200 import synth


def test_fused_layer_groups_both_stacks():
    for name, cols, qkv, gate_up in (("qwen3_4b_stack", 2560, 6144, 19456),
                                     ("llama31_8b_stack", 4096, 6144, 28672)):
        _, layer0, _, _ = synth.stack_parts(name)
        units = synth.fused_layer(layer0)
        assert [g for g, _ in units] == ["qkv", "o", "gate_up", "down"]
        parts = {g: [p.name.rsplit(".", 1)[-1] for p in ps] for g, ps in units}
        assert parts == {"qkv": ["q", "k", "v"], "o": ["o"], "gate_up": ["gate", "up"],
                         "down": ["down"]}
        rows = {g: sum(p.rows for p in ps) for g, ps in units}
        assert rows["qkv"] == qkv and rows["gate_up"] == gate_up
        assert all(ps[0].cols == cols for g, ps in units if g in ("qkv", "gate_up"))
        # Every matrix of the layer appears exactly once.
        assert sorted(p.name for _, ps in units for p in ps) == sorted(m.name for m in layer0)


def test_fused_layer_leaves_incomplete_groups_alone():
    spec = lambda n, r, c: synth.MatrixSpec(f"layers.0.{n}", r, c, "normal", 0.02, 0)  # noqa: E731
    units = synth.fused_layer([spec("q", 8, 64), spec("k", 8, 64), spec("o", 8, 64)])
    assert [g for g, _ in units] == ["q", "k", "o"]
    with pytest.raises(ValueError):
        synth.fused_layer([spec("gate", 8, 64), spec("up", 8, 128)])


def test_stacked_matrix_and_oracle_gemv(orc):
    parts = [synth.MatrixSpec(f"layers.0.{n}", r, 200, "normal", 0.02, t)
             for t, (n, r) in enumerate((("q", 24), ("k", 9), ("v", 9)))]
    w = synth.stacked_matrix(parts, 5)
    split = np.cumsum([0] + [p.rows for p in parts])
    for i, p in enumerate(parts):
        assert np.array_equal(w[split[i]:split[i + 1]], synth.matrix(p, 5))
    assert np.array_equal(orc.decode(orc.encode(w)), w)
    x = synth.activations(5, 3, 200)
    y = orc.gemv(w, x)
    for i, p in enumerate(parts):  # FP64 sums of the same terms: identical
        assert np.array_equal(y[:, split[i]:split[i + 1]], orc.gemv(synth.matrix(p, 5), x))


def test_binding_split_and_checks(monkeypatch):
    torch = pytest.importorskip("torch")
    from lossless_bf16_weight_nwc_b200 import build
    build.build()
    from lossless_bf16_weight_nwc_b200 import _lib
    with pytest.raises(ValueError):
        _lib.CompressedMatrix.compress_fused([np.zeros((8, 64), np.uint16),
                                              np.zeros((8, 32), np.uint16)])
    with pytest.raises(ValueError):
        _lib.CompressedMatrix.compress_fused([])
    monkeypatch.setattr(_lib, "nwc_handle_destroy", lambda h: None)
    m = _lib.CompressedMatrix(torch.empty(256, dtype=torch.uint8, device="meta"), object(),
                              42, 64, 256)
    y = torch.arange(2 * 42, dtype=torch.float32).reshape(2, 42)
    assert [t.shape[-1] for t in m.split(y)] == [42]
    m.row_splits = [0, 24, 33, 42]
    parts = m.split(y)
    assert [t.shape for t in parts] == [(2, 24), (2, 9), (2, 9)]
    assert torch.equal(torch.cat(parts, dim=1), y)
