"""Per-shape choice of the compressed format by measurement.

"Unweight: how we compressed an LLM 22% without sacrificing quality", section
"Direct GPU Decompression": the execution strategy depends on the weight
matrix and the batch size, and an autotuner picks the fastest one for each
workload.  Here the strategies are the format's tile width (64, 128, 256 or
512 columns: how many tiles, and so how the persistent CTAs and the split-K
reduction divide a matrix) and its code limit (7 bits, whose 14-bit peek always
holds two codes, or a longer limit).  Both are fixed when a matrix is
compressed, so `tune` compresses the matrix once per candidate, times its GEMV
at the given batch on the current device with CUDA events, and returns the
fastest.  Choices are remembered per (device, rows, cols, batch), the
quantities they depend on (the values move the compressed size by a few per
cent at most).

Every timed call runs the library's kernels; this module only chooses among
them.
"""
from __future__ import annotations

import dataclasses
import json
import os
from typing import Callable, Iterable, Sequence

import numpy as np

# (tile_cols, lmax): lmax 0 is the library's automatic limit (7 unless the
# matrix holds more than 128 distinct exponents).
DEFAULT_CANDIDATES: tuple[tuple[int, int], ...] = ((512, 0), (256, 0), (128, 0), (512, 12))
TILE_COLS = (64, 128, 256, 512)


@dataclasses.dataclass(frozen=True)
class Choice:
    tile_cols: int
    lmax: int
    us_per_call: float
    timings: dict  # "tile_cols/lmax" -> microseconds per call


def _key(device_name: str, rows: int, cols: int, batch: int) -> str:
    return f"{device_name}|{rows}x{cols}|b{batch}"


def validate_candidates(candidates: Iterable[Sequence[int]]) -> list[tuple[int, int]]:
    out = []
    for cand in candidates:
        tile_cols, lmax = int(cand[0]), int(cand[1])
        if tile_cols not in TILE_COLS:
            raise ValueError(f"tile_cols {tile_cols}: one of {TILE_COLS}")
        if not 0 <= lmax <= 12:
            raise ValueError(f"lmax {lmax}: 0 (automatic) or 1..12")
        if (tile_cols, lmax) not in out:
            out.append((tile_cols, lmax))
    if not out:
        raise ValueError("no candidates")
    return out


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
                 activations: Callable[[int, int], object] | None = None):
        """compress(w, tile_cols, lmax), timer(matrix, x, reps) -> microseconds,
        device_name() and activations(batch, cols) default to the library, CUDA
        events, the current CUDA device and seeded BF16 activations on it."""
        self.path = path
        self.cache: dict[str, dict] = {}
        if path and os.path.exists(path):
            with open(path) as f:
                self.cache = json.load(f)
        self._compress = compress
        self._timer = timer
        self._device_name = device_name
        self._make_x = activations

    def _name(self) -> str:
        if self._device_name is not None:
            return self._device_name()
        import torch
        return torch.cuda.get_device_name()

    def lookup(self, rows: int, cols: int, batch: int) -> Choice | None:
        hit = self.cache.get(_key(self._name(), rows, cols, batch))
        return None if hit is None else Choice(**hit)

    def tune(self, w_host: np.ndarray, batch: int, candidates=DEFAULT_CANDIDATES,
             reps: int = 50, retune: bool = False) -> Choice:
        """The fastest candidate for this matrix shape and batch on the current
        device (from the cache unless retune)."""
        w_host = np.ascontiguousarray(w_host, dtype=np.uint16)
        if w_host.ndim != 2:
            raise ValueError("w_host: a 2-D matrix of BF16 bit patterns")
        if not 1 <= batch <= 64:
            raise ValueError("batch: 1..64")
        rows, cols = w_host.shape
        key = _key(self._name(), rows, cols, batch)
        if not retune and key in self.cache:
            return Choice(**self.cache[key])
        cands = validate_candidates(candidates)
        compress = self._compress or self._compress_default
        timer = self._timer or time_gemv
        x = self._activations(batch, cols)
        timings, refused = {}, {}
        for tile_cols, lmax in cands:
            try:
                m = compress(w_host, tile_cols=tile_cols, lmax=lmax)
            except RuntimeError as e:  # e.g. a code limit too short for the matrix
                refused[f"{tile_cols}/{lmax}"] = str(e)
                continue
            try:
                timings[f"{tile_cols}/{lmax}"] = float(timer(m, x, reps))
            finally:
                close = getattr(m, "close", None)
                if close:
                    close()
        if not timings:
            raise RuntimeError(f"no candidate could be compressed: {refused}")
        timed = [c for c in cands if f"{c[0]}/{c[1]}" in timings]
        # Fastest; on a tie the wider tile, then the automatic code limit.
        best = min(timed, key=lambda c: (timings[f"{c[0]}/{c[1]}"], -c[0], c[1]))
        choice = Choice(best[0], best[1], timings[f"{best[0]}/{best[1]}"], timings)
        self.cache[key] = dataclasses.asdict(choice)
        if self.path:
            with open(self.path, "w") as f:
                json.dump(self.cache, f, indent=1, sort_keys=True)
        return choice

    def _activations(self, batch: int, cols: int):
        if self._make_x is not None:
            return self._make_x(batch, cols)
        import torch
        from . import synth
        x = synth.activations(0, batch, cols)
        return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()

    @staticmethod
    def _compress_default(w_host, tile_cols, lmax):
        from ._lib import CompressedMatrix
        return CompressedMatrix.compress(w_host, tile_cols=tile_cols, lmax=lmax)
