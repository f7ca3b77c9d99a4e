"""Seeded synthetic inputs: BF16 weight matrices and activations.

This module only draws random numbers; it holds none of the compression
arithmetic, and both the tests' oracle side and the CUDA side take their inputs
from it.  Every value is a pure function of (seed, tensor id, element index), so
any row of any matrix can be regenerated on its own:

* uniform(seed, tensor, c) = (m(key + (c + 1) * G) >> 11 + 0.5) * 2**-53, where
  m is the SplitMix64 output function (Steele, Lea & Flood, "Fast splittable
  pseudorandom number generators", 2014), G = 0x9E3779B97F4A7C15 and
  key = m(seed * 2**32 + tensor);
* normal draw d of element e uses the Box-Muller transform (1958) of the uniforms
  with counters 2 (e D + d) and 2 (e D + d) + 1, D draws per element;
* values are formed in float64, rounded to float32, then to BF16 with
  round-to-nearest-even.

The workloads follow the benchmark configurations: a 1024^2 matrix, a 4096^2
matrix with 0.1 % outliers, an MLP pair with Student-t(5) entries, and
Qwen3-4B- and Llama-3.1-8B-shaped weight stacks (random init, no checkpoints).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

_G = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
X_TENSOR = 0xFFFF          # tensor id of the activations x
SCALE_TENSOR = 0xFFFE      # tensor id of per-row scales (Llama-shaped stack)


def _mix(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.uint64, copy=True)
    with np.errstate(over="ignore"):
        z ^= z >> np.uint64(30)
        z *= _M1
        z ^= z >> np.uint64(27)
        z *= _M2
        z ^= z >> np.uint64(31)
    return z


def _key(seed: int, tensor: int) -> np.uint64:
    k = np.array([(seed << 32) + tensor], dtype=np.uint64)
    return _mix(k)[0]


def uniform(seed: int, tensor: int, counters: np.ndarray) -> np.ndarray:
    """U(0,1) float64, never 0 or 1, for the given counters (uint64 array)."""
    c = np.asarray(counters, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = _key(seed, tensor) + (c + np.uint64(1)) * _G
    bits = _mix(z) >> np.uint64(11)
    return (bits.astype(np.float64) + 0.5) * (2.0 ** -53)


def normal(seed: int, tensor: int, elements: np.ndarray, draws: int = 1,
           draw: int = 0) -> np.ndarray:
    """Standard normal float64 for draw `draw` of each element."""
    e = np.asarray(elements, dtype=np.uint64)
    base = (e * np.uint64(draws) + np.uint64(draw)) * np.uint64(2)
    u1 = uniform(seed, tensor, base)
    u2 = uniform(seed, tensor, base + np.uint64(1))
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


def to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """float -> float32 -> BF16 bit patterns (round to nearest, ties to even)."""
    f = np.asarray(v, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    rounded = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    out = rounded.astype(np.uint16)
    nan = np.isnan(f)
    if nan.any():
        out[nan] = (u[nan] >> np.uint64(16)).astype(np.uint16) | np.uint16(0x40)
    return out


def bf16_bits_to_float(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------
# Matrix kinds
# --------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class MatrixSpec:
    name: str
    rows: int           # output features
    cols: int           # input features
    kind: str           # "normal", "normal_outliers", "student_t5", "normal_rowscale"
    std: float
    tensor: int         # tensor id inside the workload's seed

    @property
    def weights(self) -> int:
        return self.rows * self.cols


def _values(spec: MatrixSpec, seed: int, row_begin: int, row_end: int) -> np.ndarray:
    cols = spec.cols
    e = np.arange(row_begin * cols, row_end * cols, dtype=np.uint64)
    if spec.kind == "normal":
        v = spec.std * normal(seed, spec.tensor, e)
    elif spec.kind == "normal_outliers":
        # 0.1 % of positions (an extra uniform below 1e-3) are scaled by 20.
        v = spec.std * normal(seed, spec.tensor, e, draws=2, draw=0)
        u = uniform(seed, spec.tensor, e * np.uint64(4) + np.uint64(2))
        v = np.where(u < 1e-3, v * 20.0, v)
    elif spec.kind == "student_t5":
        # t(5) = Z / sqrt(chi2_5 / 5); variance 5/3, rescaled to the target std.
        z = normal(seed, spec.tensor, e, draws=6, draw=0)
        chi2 = np.zeros_like(z)
        for d in range(1, 6):
            chi2 += normal(seed, spec.tensor, e, draws=6, draw=d) ** 2
        v = spec.std / math.sqrt(5.0 / 3.0) * z / np.sqrt(chi2 / 5.0)
    elif spec.kind == "normal_rowscale":
        # Per-output-channel scale s_n ~ LogNormal(0, 0.5).
        rows = np.arange(row_begin, row_end, dtype=np.uint64)
        s = np.exp(0.5 * normal(seed, SCALE_TENSOR * 65536 + spec.tensor, rows))
        v = spec.std * normal(seed, spec.tensor, e) * np.repeat(s, cols)
    else:
        raise ValueError(spec.kind)
    return v


def matrix(spec: MatrixSpec, seed: int, row_begin: int = 0,
           row_end: int | None = None, chunk_rows: int | None = None) -> np.ndarray:
    """BF16 bit patterns of rows [row_begin, row_end) of a matrix, uint16 [r, cols]."""
    row_end = spec.rows if row_end is None else row_end
    out = np.empty((row_end - row_begin, spec.cols), dtype=np.uint16)
    step = chunk_rows or max(1, (1 << 22) // spec.cols)
    for r0 in range(row_begin, row_end, step):
        r1 = min(row_end, r0 + step)
        out[r0 - row_begin:r1 - row_begin] = to_bf16_bits(
            _values(spec, seed, r0, r1)).reshape(r1 - r0, spec.cols)
    return out


def activations(seed: int, batch: int, cols: int, tensor: int = X_TENSOR) -> np.ndarray:
    """x ~ N(0, 1) as BF16 bit patterns, [batch, cols]; row b is the same for any batch."""
    e = np.arange(batch * cols, dtype=np.uint64)
    return to_bf16_bits(normal(seed, tensor, e)).reshape(batch, cols)


# --------------------------------------------------------------------------
# Workloads
# --------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    matrices: tuple
    batches: tuple
    description: str

    @property
    def weights(self) -> int:
        return sum(m.weights for m in self.matrices)


def _stack(prefix_layers: int, shapes, extra, kind: str, std: float):
    mats = []
    tid = 0
    for layer in range(prefix_layers):
        for nm, (r, c) in shapes:
            mats.append(MatrixSpec(f"layers.{layer}.{nm}", r, c, kind, std, tid))
            tid += 1
    for nm, (r, c) in extra:
        mats.append(MatrixSpec(nm, r, c, kind, std, tid))
        tid += 1
    return tuple(mats)


def workload(name: str) -> Workload:
    if name == "single_1024":
        return Workload(name, 0, (MatrixSpec("w", 1024, 1024, "normal", 0.02, 0),),
                        (1,), "1024x1024, N(0, 0.02), x ~ N(0, 1), seed 0")
    if name == "attn_4096_outliers":
        return Workload(name, 1, (MatrixSpec("w", 4096, 4096, "normal_outliers",
                                             1.0 / 64.0, 0),),
                        (1, 4), "4096x4096, N(0, 1/64) with 0.1 % of entries x20, seed 1")
    if name == "mlp_pair_t5":
        return Workload(name, 2, (MatrixSpec("up", 14336, 4096, "student_t5", 0.015, 0),
                                  MatrixSpec("down", 4096, 14336, "student_t5", 0.015, 1)),
                        (1, 2, 8), "MLP pair 14336x4096 + 4096x14336, Student-t(5) std 0.015, seed 2")
    if name == "qwen3_4b_stack":
        shapes = [("q", (4096, 2560)), ("k", (1024, 2560)), ("v", (1024, 2560)),
                  ("o", (2560, 4096)), ("gate", (9728, 2560)), ("up", (9728, 2560)),
                  ("down", (2560, 9728))]
        return Workload(name, 3, _stack(36, shapes, [("lm_head", (151936, 2560))],
                                        "normal", 0.02),
                        (1,), "Qwen3-4B-shaped stack: 36 layers + tied 151936x2560 lm_head, N(0, 0.02), seed 3")
    if name == "llama31_8b_stack":
        shapes = [("q", (4096, 4096)), ("k", (1024, 4096)), ("v", (1024, 4096)),
                  ("o", (4096, 4096)), ("gate", (14336, 4096)), ("up", (14336, 4096)),
                  ("down", (4096, 14336))]
        return Workload(name, 4, _stack(32, shapes, [("lm_head", (128256, 4096))],
                                        "normal_rowscale", 0.02),
                        (1, 16, 64), "Llama-3.1-8B-shaped stack: 32 layers + 128256x4096 lm_head, "
                        "N(0, 0.02) x LogNormal(0, 0.5) row scale, seed 4")
    raise KeyError(name)


# The stacks' per-token sequences reuse one generated layer for every layer
# (a layer of either stack is larger than B200's L2, so each is read cold), and
# build the lm_head from its first HEAD_BLOCK_ROWS rows repeated down the
# matrix: full shapes at a fraction of the generation time.
HEAD_BLOCK_ROWS = 16384


def stack_parts(name: str):
    """(workload, the 7 matrices of layer 0, the lm_head spec, number of layers)."""
    wl = workload(name)
    layer0 = [m for m in wl.matrices if m.name.startswith("layers.0.")]
    head = [m for m in wl.matrices if m.name == "lm_head"][0]
    layers = len({m.name.split(".")[1] for m in wl.matrices if m.name.startswith("layers.")})
    return wl, layer0, head, layers


# Projections of a layer that read the same input, run as one matrix whose rows
# are the parts' rows in this order ("NWC — Neural Weight Compression",
# "Install": fuse(model) before convert(model); "Run a model": --fusion).
FUSED_GROUPS = (("qkv", ("q", "k", "v")), ("gate_up", ("gate", "up")))


def fused_layer(layer: list[MatrixSpec]) -> list[tuple[str, list[MatrixSpec]]]:
    """A layer's matrices as (name, parts) in layer order: each group of
    FUSED_GROUPS present in the layer becomes one entry at the place of its first
    part; every other matrix stands alone."""
    by_short = {m.name.rsplit(".", 1)[-1]: m for m in layer}
    group_of = {part: (g, parts) for g, parts in FUSED_GROUPS
                if all(p in by_short for p in parts) for part in parts}
    out, done = [], set()
    for m in layer:
        short = m.name.rsplit(".", 1)[-1]
        if short not in group_of:
            out.append((short, [m]))
            continue
        g, parts = group_of[short]
        if g in done:
            continue
        members = [by_short[p] for p in parts]
        if len({p.cols for p in members}) != 1:
            raise ValueError(f"{g}: parts read inputs of different widths")
        out.append((g, members))
        done.add(g)
    return out


def stacked_matrix(parts: list[MatrixSpec], seed: int) -> np.ndarray:
    """The parts' generated matrices with their rows stacked in order."""
    return np.ascontiguousarray(np.concatenate([matrix(p, seed) for p in parts], axis=0))


def head_matrix(spec: MatrixSpec, seed: int) -> np.ndarray:
    """The lm_head as its first HEAD_BLOCK_ROWS generated rows, repeated."""
    block = matrix(spec, seed, 0, min(HEAD_BLOCK_ROWS, spec.rows))
    reps = -(-spec.rows // block.shape[0])
    return np.ascontiguousarray(np.tile(block, (reps, 1))[:spec.rows])


WORKLOADS = ("single_1024", "attn_4096_outliers", "mlp_pair_t5", "qwen3_4b_stack",
             "llama31_8b_stack")
