"""Per-shape choice of the GEMV strategy by measurement.

"Unweight: how we compressed an LLM 22% without sacrificing quality", section
"Direct GPU Decompression": the execution strategy depends on the weight
matrix and the batch size, and an autotuner picks the fastest one for each
workload.  Here a strategy is

* the format, fixed when a matrix is compressed: the tile width (64, 128, 256
  or 512 columns: how many tiles, and so how the persistent CTAs divide a
  matrix), the code limit (7 bits, whose 14-bit table peek always holds two
  codes, or a longer limit), the bit streams per lane (1, or 2 so that a lane
  follows two independent decode chains) and the exponent code (the
  length-limited prefix code, the table-free ranked unary code, or the prefix
  code of the 16 most frequent exponents with verbatim runs for the rest);
* the kernel, chosen per call: the CUDA-core kernel (mma.sync on the decoded
  registers, up to 16 rows of x per launch, the matrix decoded again for every
  16 rows) or the tensor-core kernel (tcgen05, each weight decoded once into
  shared memory for up to 64 rows of x).

`tune` compresses the matrix once per format, times its GEMV at the given batch
under each kernel on the current device with CUDA events behind an L2 flush,
and returns the fastest.  Choices are remembered per (device, rows, cols,
batch), the quantities they depend on (the values move the compressed size by
a few per cent at most).  `apply` sets a compressed matrix's kernel threshold
from a choice.

Every timed call runs the library's kernels; this module only chooses among
them.
"""
from __future__ import annotations

import dataclasses
import json
import os
from typing import Callable, Iterable

import numpy as np

TILE_COLS = (64, 128, 256, 512)
CODES = ("prefix", "rank", "escape")
KERNELS = ("cuda", "tensor")


@dataclasses.dataclass(frozen=True)
class Strategy:
    tile_cols: int = 512
    lmax: int = 0          # prefix: 0 = automatic (7 unless > 128 exponents); rank: ranks
                           # (0 = 7); escape: 0 = 7, else 1..7
    streams: int = 1
    code: str = "prefix"
    kernel: str = "cuda"

    @property
    def key(self) -> str:
        return f"{self.tile_cols}/{self.lmax}/{self.streams}/{self.code}/{self.kernel}"

    @property
    def format(self) -> tuple:
        return (self.tile_cols, self.lmax, self.streams, self.code)


def default_candidates(batch: int) -> list[Strategy]:
    """The formats worth comparing, each under the kernels that suit the batch
    (the tensor-core kernel for any batch; the CUDA-core one up to 16 rows of x
    per launch, so for larger batches only as a baseline)."""
    formats = [(512, 0, 1, "prefix"), (512, 0, 2, "prefix"), (256, 0, 1, "prefix"),
               (512, 12, 1, "prefix"), (512, 0, 1, "rank"), (512, 0, 1, "escape")]
    kernels = ("cuda", "tensor") if batch >= 8 else ("cuda",)
    return [Strategy(*f, kernel=k) for f in formats for k in kernels]


@dataclasses.dataclass(frozen=True)
class Choice:
    strategy: Strategy
    us_per_call: float
    timings: dict  # Strategy.key -> microseconds per call

    def to_json(self) -> dict:
        return {"strategy": dataclasses.asdict(self.strategy), "us_per_call": self.us_per_call,
                "timings": self.timings}

    @classmethod
    def from_json(cls, d: dict) -> "Choice":
        return cls(Strategy(**d["strategy"]), float(d["us_per_call"]), dict(d["timings"]))


def _key(device_name: str, rows: int, cols: int, batch: int) -> str:
    return f"{device_name}|{rows}x{cols}|b{batch}"


def validate_candidates(candidates: Iterable[Strategy]) -> list[Strategy]:
    out = []
    for s in candidates:
        if not isinstance(s, Strategy):
            raise TypeError(f"{s!r}: expected a Strategy")
        if s.tile_cols not in TILE_COLS:
            raise ValueError(f"tile_cols {s.tile_cols}: one of {TILE_COLS}")
        if s.code not in CODES:
            raise ValueError(f"code {s.code!r}: one of {CODES}")
        if s.kernel not in KERNELS:
            raise ValueError(f"kernel {s.kernel!r}: one of {KERNELS}")
        if s.streams not in (1, 2) or (s.code != "prefix" and s.streams != 1):
            raise ValueError(f"streams {s.streams}: 1 or 2 (1 for the rank and escape codes)")
        if not 0 <= s.lmax <= (12 if s.code == "prefix" else 7):
            raise ValueError(f"lmax {s.lmax}: 0 (automatic) or 1..12 (rank, escape: 1..7)")
        if s not in out:
            out.append(s)
    if not out:
        raise ValueError("no candidates")
    return out


def apply(m, strategy: Strategy) -> None:
    """Make a compressed matrix's GEMVs take the strategy's kernel: the
    tensor-core kernel for every batch, or never."""
    from ._lib import nwc_gemv_set_tc_min_batch
    nwc_gemv_set_tc_min_batch(m.handle, 1 if strategy.kernel == "tensor" else 0)


def time_gemv(m, x, reps: int = 50, flush_bytes: int = 256 << 20) -> float:
    """Microseconds per GEMV call on the current stream, timed with CUDA events
    around each call; a buffer larger than B200's L2 is overwritten before each
    call so the weights are read from HBM, as in a model's layer sequence."""
    import torch
    y = torch.empty((x.shape[0], m.rows), dtype=torch.float32, device=x.device)
    flush = torch.empty(flush_bytes, dtype=torch.uint8, device=x.device)
    for _ in range(3):
        m.gemv(x, y)
    stream = torch.cuda.current_stream()
    events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(reps)]
    for start, end in events:
        flush.zero_()
        start.record(stream)
        m.gemv(x, y)
        end.record(stream)
    torch.cuda.synchronize()
    return 1e3 * float(np.median([s.elapsed_time(e) for s, e in events]))


class Tuner:
    """Remembers choices per (device, rows, cols, batch); optionally in a JSON file."""

    def __init__(self, path: str | None = None,
                 compress: Callable | None = None, timer: Callable | None = None,
                 device_name: Callable[[], str] | None = None,
                 activations: Callable[[int, int], object] | None = None,
                 set_kernel: Callable | None = None):
        """compress(w, strategy) -> matrix, timer(matrix, x, reps) ->
        microseconds, set_kernel(matrix, strategy), device_name() and
        activations(batch, cols) default to the library, CUDA events, the
        current CUDA device and seeded BF16 activations on it."""
        self.path = path
        self.cache: dict[str, dict] = {}
        if path and os.path.exists(path):
            with open(path) as f:
                self.cache = json.load(f)
        self._compress = compress
        self._timer = timer
        self._device_name = device_name
        self._make_x = activations
        self._set_kernel = set_kernel

    def _name(self) -> str:
        if self._device_name is not None:
            return self._device_name()
        import torch
        return torch.cuda.get_device_name()

    def lookup(self, rows: int, cols: int, batch: int) -> Choice | None:
        hit = self.cache.get(_key(self._name(), rows, cols, batch))
        return None if hit is None else Choice.from_json(hit)

    def tune(self, w_host: np.ndarray, batch: int, candidates: Iterable[Strategy] | None = None,
             reps: int = 50, retune: bool = False) -> Choice:
        """The fastest candidate for this matrix shape and batch on the current
        device (from the cache unless retune)."""
        return self.tune_batches(w_host, [batch], candidates, reps, retune)[batch]

    def tune_batches(self, w_host: np.ndarray, batches: Iterable[int],
                     candidates: Iterable[Strategy] | None = None, reps: int = 50,
                     retune: bool = False) -> dict:
        """tune for several batches at once: each format is compressed once and
        timed at every batch that is not cached yet.  Returns {batch: Choice}."""
        w_host = np.ascontiguousarray(w_host, dtype=np.uint16)
        if w_host.ndim != 2:
            raise ValueError("w_host: a 2-D matrix of BF16 bit patterns")
        batches = list(dict.fromkeys(int(b) for b in batches))
        if not batches or not all(1 <= b <= 64 for b in batches):
            raise ValueError("batch: 1..64")
        rows, cols = w_host.shape
        name = self._name()
        out, todo = {}, []
        for b in batches:
            key = _key(name, rows, cols, b)
            if not retune and key in self.cache:
                out[b] = Choice.from_json(self.cache[key])
            else:
                todo.append(b)
        if not todo:
            return out
        cands = {b: validate_candidates(default_candidates(b) if candidates is None
                                        else candidates) for b in todo}
        compress = self._compress or self._compress_default
        timer = self._timer or time_gemv
        set_kernel = self._set_kernel or apply
        xs = {b: self._activations(b, cols) for b in todo}
        timings = {b: {} for b in todo}
        refused = {}
        formats: dict[tuple, list[Strategy]] = {}
        for b in todo:
            for st in cands[b]:
                formats.setdefault(st.format, [])
                if st not in formats[st.format]:
                    formats[st.format].append(st)
        for fmt, strategies in formats.items():
            try:
                m = compress(w_host, strategies[0])
            except RuntimeError as e:  # e.g. a code limit too short for the matrix
                for st in strategies:
                    refused[st.key] = str(e)
                continue
            try:
                for b in todo:
                    for st in strategies:
                        if st in cands[b]:
                            set_kernel(m, st)
                            timings[b][st.key] = float(timer(m, xs[b], reps))
            finally:
                close = getattr(m, "close", None)
                if close:
                    close()
        for b in todo:
            if not timings[b]:
                raise RuntimeError(f"no candidate could be compressed: {refused}")
            timed = [st for st in cands[b] if st.key in timings[b]]
            # Fastest; on a tie the earlier candidate (the simpler format first).
            best = min(timed, key=lambda st: (timings[b][st.key], timed.index(st)))
            out[b] = Choice(best, timings[b][best.key], timings[b])
            self.cache[_key(name, rows, cols, b)] = out[b].to_json()
        if self.path:
            with open(self.path, "w") as f:
                json.dump(self.cache, f, indent=1, sort_keys=True)
        return out

    def _activations(self, batch: int, cols: int):
        if self._make_x is not None:
            return self._make_x(batch, cols)
        import torch
        from . import synth
        x = synth.activations(0, batch, cols)
        return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()

    @staticmethod
    def _compress_default(w_host, s: Strategy):
        from ._lib import NWC_CODE_ESCAPE, NWC_CODE_PREFIX, NWC_CODE_RANK, CompressedMatrix
        code = {"prefix": NWC_CODE_PREFIX, "rank": NWC_CODE_RANK, "escape": NWC_CODE_ESCAPE}
        return CompressedMatrix.compress(w_host, tile_cols=s.tile_cols, lmax=s.lmax,
                                         streams=s.streams, code=code[s.code])


def sweep(workloads, batches, path: str, reps: int = 30) -> dict:
    """Tunes every distinct matrix shape of the given workloads (synthetic
    weights of the workload's distribution) at each batch; returns and saves
    the cache."""
    from . import synth
    tuner = Tuner(path)
    for name in workloads:
        if name in ("qwen3_4b_stack", "llama31_8b_stack"):
            wl, layer0, head, _ = synth.stack_parts(name)
            specs = layer0 + [head]
        else:
            wl = synth.workload(name)
            head, specs = None, list(wl.matrices)
        seen = set()
        for spec in specs:
            if (spec.rows, spec.cols) in seen:
                continue
            seen.add((spec.rows, spec.cols))
            w = synth.head_matrix(spec, wl.seed) if spec is head else synth.matrix(spec, wl.seed)
            for batch, c in tuner.tune_batches(w, batches, reps=reps).items():
                print(f"{name} {spec.rows}x{spec.cols} b{batch}: {c.strategy.key} "
                      f"{c.us_per_call:.2f} us", flush=True)
    return tuner.cache


if __name__ == "__main__":
    import argparse
    ap = argparse.ArgumentParser(description="tune the GEMV strategy per matrix shape and batch")
    ap.add_argument("--workloads", nargs="+", default=["qwen3_4b_stack", "llama31_8b_stack"])
    ap.add_argument("--batches", nargs="+", type=int, default=[1, 16, 64])
    ap.add_argument("--out", required=True, help="the JSON cache to write (and extend)")
    ap.add_argument("--reps", type=int, default=30)
    a = ap.parse_args()
    sweep(a.workloads, a.batches, a.out, a.reps)
