"""The format autotuner's host logic on the CPU, with a stand-in compressor and
timer: it picks the fastest candidate (wider tile, then automatic code limit on
a tie), skips candidates that cannot be compressed, remembers choices per
(device, rows, cols, batch) in memory and in a JSON file, and checks its
arguments."""
import numpy as np
import pytest

from lossless_bf16_weight_nwc_b200 import autotune


class Fake:
    def __init__(self, times, refuse=()):
        self.times, self.refuse, self.compressed, self.closed = times, set(refuse), [], 0

    def compress(self, w, tile_cols, lmax):
        if (tile_cols, lmax) in self.refuse:
            raise RuntimeError("nwc_plan failed: NWC_ERR_INVALID_ARG")
        self.compressed.append((tile_cols, lmax))
        fake = self

        class M:
            key = (tile_cols, lmax)

            def close(self):
                fake.closed += 1
        return M()

    def timer(self, m, x, reps):
        assert x.shape[0] in (1, 4) and reps == 7
        return self.times[m.key]


def tuner(fake, path=None, name="B200"):
    return autotune.Tuner(path, compress=fake.compress, timer=fake.timer, device_name=lambda: name,
                          activations=lambda b, k: np.zeros((b, k), dtype=np.uint16))


W = np.zeros((40, 1000), dtype=np.uint16)


def test_picks_the_fastest_and_remembers(tmp_path):
    fake = Fake({(512, 0): 30.0, (256, 0): 21.5, (128, 0): 25.0, (512, 12): 40.0})
    t = tuner(fake, str(tmp_path / "tune.json"))
    c = t.tune(W, 1, reps=7)
    assert (c.tile_cols, c.lmax, c.us_per_call) == (256, 0, 21.5)
    assert c.timings == {"512/0": 30.0, "256/0": 21.5, "128/0": 25.0, "512/12": 40.0}
    assert fake.closed == 4
    t.tune(W, 1, reps=7)                                   # cached: nothing compressed again
    assert len(fake.compressed) == 4
    assert t.lookup(40, 1000, 1) == c and t.lookup(40, 1000, 4) is None
    again = tuner(Fake({}), str(tmp_path / "tune.json"))   # from the file
    assert again.tune(W, 1, reps=7) == c
    other = tuner(Fake({k: 1.0 for k in fake.times}), str(tmp_path / "tune.json"), name="H100")
    assert other.tune(W, 1, reps=7).tile_cols == 512       # another device tunes anew
    t.tune(W, 1, reps=7, retune=True)
    assert len(fake.compressed) == 8


def test_ties_prefer_wider_tiles_then_automatic_limit():
    fake = Fake({(128, 0): 5.0, (512, 12): 5.0, (512, 0): 5.0})
    c = tuner(fake).tune(W, 4, candidates=[(128, 0), (512, 12), (512, 0)], reps=7)
    assert (c.tile_cols, c.lmax) == (512, 0)


def test_refused_candidates_are_skipped():
    fake = Fake({(512, 0): 9.0, (256, 0): 8.0}, refuse={(256, 0)})
    c = tuner(fake).tune(W, 1, candidates=[(512, 0), (256, 0)], reps=7)
    assert (c.tile_cols, c.timings) == (512, {"512/0": 9.0})
    with pytest.raises(RuntimeError):
        tuner(Fake({}, refuse={(512, 0)})).tune(W, 1, candidates=[(512, 0)], reps=7)


def test_arguments_checked():
    fake = Fake({})
    with pytest.raises(ValueError):
        tuner(fake).tune(W, 1, candidates=[(100, 0)])
    with pytest.raises(ValueError):
        tuner(fake).tune(W, 1, candidates=[(512, 13)])
    with pytest.raises(ValueError):
        tuner(fake).tune(W, 1, candidates=[])
    with pytest.raises(ValueError):
        tuner(fake).tune(W, 65)
    with pytest.raises(ValueError):
        tuner(fake).tune(W.reshape(-1), 1)
    assert autotune.validate_candidates([(512, 0), (512, 0), (64, 7)]) == [(512, 0), (64, 7)]
