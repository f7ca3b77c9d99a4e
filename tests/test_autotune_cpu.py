"""The strategy autotuner's host logic on the CPU, with a stand-in compressor,
timer and kernel switch: it compresses once per format and times every kernel
choice of it, picks the fastest candidate (the earlier one on a tie), skips
formats that cannot be compressed, remembers choices per (device, rows, cols,
batch) in memory and in a JSON file, and checks its arguments."""
import numpy as np
import pytest

from lossless_bf16_weight_nwc_b200 import autotune
from lossless_bf16_weight_nwc_b200.autotune import Strategy


class Fake:
    def __init__(self, times, refuse=()):
        self.times, self.refuse, self.compressed, self.closed = times, set(refuse), [], 0

    def compress(self, w, s):
        if s.format in self.refuse:
            raise RuntimeError("nwc_plan failed: NWC_ERR_INVALID_ARG")
        self.compressed.append(s.format)
        fake = self

        class M:
            fmt = s.format
            kernel = None

            def close(self):
                fake.closed += 1
        return M()

    @staticmethod
    def set_kernel(m, s):
        m.kernel = s.kernel

    def timer(self, m, x, reps):
        assert x.shape[0] in (1, 4, 16) and reps == 7
        return self.times[(*m.fmt, m.kernel)]


def tuner(fake, path=None, name="B200"):
    return autotune.Tuner(path, compress=fake.compress, timer=fake.timer, device_name=lambda: name,
                          activations=lambda b, k: np.zeros((b, k), dtype=np.uint16),
                          set_kernel=fake.set_kernel)


W = np.zeros((40, 1000), dtype=np.uint16)
A = Strategy(512, 0, 1, "prefix", "cuda")
B = Strategy(512, 0, 1, "prefix", "tensor")
C = Strategy(256, 0, 1, "prefix", "cuda")
D = Strategy(512, 0, 1, "rank", "cuda")
E = Strategy(512, 0, 2, "prefix", "tensor")


def t_of(*pairs):
    return {(*s.format, s.kernel): v for s, v in pairs}


def test_picks_the_fastest_and_remembers(tmp_path):
    fake = Fake(t_of((A, 30.0), (B, 21.5), (C, 25.0), (D, 40.0), (E, 22.0)))
    t = tuner(fake, str(tmp_path / "tune.json"))
    c = t.tune(W, 16, candidates=[A, B, C, D, E], reps=7)
    assert c.strategy == B and c.us_per_call == 21.5
    assert c.timings == {A.key: 30.0, B.key: 21.5, C.key: 25.0, D.key: 40.0, E.key: 22.0}
    assert len(fake.compressed) == 4 and fake.closed == 4   # A and B share one compression
    t.tune(W, 16, candidates=[A, B], reps=7)                # cached: nothing compressed again
    assert len(fake.compressed) == 4
    assert t.lookup(40, 1000, 16) == c and t.lookup(40, 1000, 4) is None
    again = tuner(Fake({}), str(tmp_path / "tune.json"))    # from the file
    assert again.tune(W, 16, reps=7) == c
    other = tuner(Fake(t_of((A, 1.0), (C, 1.0))), str(tmp_path / "tune.json"), name="H100")
    assert other.tune(W, 16, candidates=[A, C], reps=7).strategy == A   # another device anew
    t.tune(W, 16, candidates=[A, B, C, D, E], reps=7, retune=True)
    assert len(fake.compressed) == 8


def test_ties_prefer_the_earlier_candidate():
    fake = Fake(t_of((C, 5.0), (D, 5.0), (A, 5.0)))
    assert tuner(fake).tune(W, 4, candidates=[C, D, A], reps=7).strategy == C
    assert tuner(fake).tune(W, 4, candidates=[A, C, D], reps=7).strategy == A


def test_refused_formats_are_skipped():
    fake = Fake(t_of((A, 9.0), (B, 9.5), (C, 8.0)), refuse={C.format})
    c = tuner(fake).tune(W, 1, candidates=[A, B, C], reps=7)
    assert c.strategy == A and c.timings == {A.key: 9.0, B.key: 9.5}
    with pytest.raises(RuntimeError):
        tuner(Fake({}, refuse={A.format})).tune(W, 1, candidates=[A, B], reps=7)


def test_default_candidates_cover_the_kernels():
    small = autotune.default_candidates(1)
    large = autotune.default_candidates(16)
    assert {s.kernel for s in small} == {"cuda"}
    assert {s.kernel for s in large} == {"cuda", "tensor"}
    assert {s.code for s in large} == {"prefix", "rank", "escape"}
    assert {s.streams for s in large} == {1, 2}
    assert autotune.validate_candidates(large) == large


def test_arguments_checked():
    fake = Fake({})
    for bad in (Strategy(100), Strategy(512, 13), Strategy(512, 0, 3), Strategy(code="huffman"),
                Strategy(kernel="cpu"), Strategy(streams=2, code="rank"),
                Strategy(lmax=8, code="rank"), Strategy(streams=2, code="escape"),
                Strategy(lmax=8, code="escape")):
        with pytest.raises(ValueError):
            tuner(fake).tune(W, 1, candidates=[bad])
    with pytest.raises(TypeError):
        tuner(fake).tune(W, 1, candidates=[(512, 0)])
    with pytest.raises(ValueError):
        tuner(fake).tune(W, 1, candidates=[])
    with pytest.raises(ValueError):
        tuner(fake).tune(W, 65)
    with pytest.raises(ValueError):
        tuner(fake).tune(W.reshape(-1), 1)
    assert autotune.validate_candidates([A, A, C]) == [A, C]


def test_several_batches_share_one_compression_per_format(tmp_path):
    """tune_batches compresses each format once for all batches, times each
    batch's candidates, and caches a choice per batch; batches already cached
    are not timed again."""
    fake = Fake(t_of((A, 30.0), (B, 21.5), (C, 25.0)))
    t = tuner(fake, str(tmp_path / "tune.json"))
    got = t.tune_batches(W, [1, 16], candidates=[A, B, C], reps=7)
    assert sorted(fake.compressed) == sorted([A.format, C.format])
    assert fake.closed == 2
    assert got[1].strategy == B and got[16].strategy == B
    assert set(got[1].timings) == {A.key, B.key, C.key}
    fake.compressed.clear()
    again = t.tune_batches(W, [1, 16, 4], candidates=[A, C], reps=7)
    assert again[1] == got[1] and again[16] == got[16]
    assert again[4].strategy == C and fake.compressed == [A.format, C.format]
    with pytest.raises(ValueError):
        t.tune_batches(W, [], reps=7)
    with pytest.raises(ValueError):
        t.tune_batches(W, [65], reps=7)
