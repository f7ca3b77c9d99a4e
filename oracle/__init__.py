"""Test oracle for lossless BF16 weight compression (ctypes shim).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product library never imports it, and it imports nothing from
the product.

The arithmetic lives in ``nwc_oracle.cpp`` (plain single-threaded C++), which
states the blob format field by field and cites the page passage behind every
step.  This module only compiles it with the host C++ compiler and marshals
numpy arrays in and out.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nwc_oracle.cpp")
_HDR = os.path.join(_HERE, "nwc_oracle.h")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_handle = None

ORC_OK = 0
ORC_E_ARG = -1
ORC_E_SPACE = -2
ORC_E_CORRUPT = -3
ORC_E_LMAX = -4


class OracleError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: oracle status {code}")
        self.code = code


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source when missing or stale."""
    stale = force or not os.path.exists(_LIB)
    if not stale:
        t = os.path.getmtime(_LIB)
        stale = t < os.path.getmtime(_SRC) or t < os.path.getmtime(_HDR)
    if stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-Wall", "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def _declare(h: ctypes.CDLL) -> ctypes.CDLL:
    """Declare argument types of every exported oracle function."""
    c = ctypes
    i64, u8p, u16p = c.c_int64, c.POINTER(c.c_uint8), c.POINTER(c.c_uint16)
    h.orc_plane_split.argtypes = [c.c_uint16, u8p, u8p]
    h.orc_plane_split.restype = None
    h.orc_plane_join.argtypes = [c.c_uint8, c.c_uint8]
    h.orc_plane_join.restype = c.c_uint16
    h.orc_histogram.argtypes = [u16p, i64, i64, c.POINTER(c.c_uint64)]
    h.orc_code_lengths.argtypes = [c.POINTER(c.c_uint64), c.c_int, u8p]
    h.orc_canonical_codes.argtypes = [u8p, c.POINTER(c.c_uint32)]
    h.orc_blob_size.argtypes = [u16p, i64, i64, c.c_int, c.c_int, c.c_int,
                                c.POINTER(i64)]
    h.orc_encode.argtypes = [u16p, i64, i64, c.c_int, c.c_int, c.c_int, u8p,
                             i64, c.POINTER(i64)]
    h.orc_blob_size_streams.argtypes = [u16p, i64, i64, c.c_int, c.c_int, c.c_int, c.c_int,
                                        c.POINTER(i64)]
    h.orc_encode_streams.argtypes = [u16p, i64, i64, c.c_int, c.c_int, c.c_int, c.c_int, u8p,
                                     i64, c.POINTER(i64)]
    h.orc_blob_info.argtypes = [u8p, i64, c.POINTER(i64), c.POINTER(i64)]
    h.orc_decode.argtypes = [u8p, i64, u16p, i64]
    h.orc_decode_tiles.argtypes = [u8p, i64, i64, i64, u16p, i64]
    h.orc_gemv.argtypes = [u16p, i64, i64, u16p, c.c_int, i64, i64,
                           c.POINTER(c.c_double)]
    h.orc_rank_table.argtypes = [u16p, i64, i64, c.c_int, c.c_int, c.c_int, u8p,
                                 c.POINTER(c.c_int)]
    h.orc_rank_blob_size.argtypes = [u16p, i64, i64, c.c_int, c.c_int, c.c_int,
                                     c.POINTER(i64)]
    h.orc_rank_encode.argtypes = [u16p, i64, i64, c.c_int, c.c_int, c.c_int, u8p,
                                  i64, c.POINTER(i64)]
    h.orc_rank_decode.argtypes = [u8p, i64, u16p, i64]
    h.orc_escape_blob_size.argtypes = [u16p, i64, i64, c.c_int, c.c_int, c.c_int, c.c_int,
                                       c.POINTER(i64)]
    h.orc_escape_encode.argtypes = [u16p, i64, i64, c.c_int, c.c_int, c.c_int, c.c_int, u8p,
                                    i64, c.POINTER(i64)]
    h.orc_escape_decode.argtypes = [u8p, i64, u16p, i64]
    return h


def lib() -> ctypes.CDLL:
    global _handle
    with _lock:
        if _handle is None:
            build()
            _handle = _declare(ctypes.CDLL(_LIB))
    return _handle


class use_library:
    """Route this module's functions through another build of the oracle source
    (used by the mutation tests, which compile planted mistakes on the CPU)."""

    def __init__(self, path: str):
        self._lib = _declare(ctypes.CDLL(path))

    def __enter__(self):
        global _handle
        lib()
        self._saved = _handle
        _handle = self._lib
        return self

    def __exit__(self, *exc):
        global _handle
        _handle = self._saved
        return False


def source() -> str:
    with open(_SRC) as f:
        return f.read()


def compile_variant(src_text: str, out_path: str) -> str:
    """Compile an edited copy of the oracle source into out_path."""
    cpp = out_path + ".cpp"
    with open(cpp, "w") as f:
        f.write(src_text)
    subprocess.check_call(["g++", "-O1", "-std=c++17", "-shared", "-fPIC", "-I", _HERE,
                           "-o", out_path, cpp])
    return out_path


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def _check(rc: int, what: str) -> None:
    if rc != ORC_OK:
        raise OracleError(rc, what)


def plane_split(w: int) -> tuple[int, int]:
    s, r = ctypes.c_uint8(), ctypes.c_uint8()
    lib().orc_plane_split(w, ctypes.byref(s), ctypes.byref(r))
    return s.value, r.value


def plane_join(s: int, r: int) -> int:
    return int(lib().orc_plane_join(s, r))


def histogram(w: np.ndarray) -> np.ndarray:
    w = np.ascontiguousarray(w, dtype=np.uint16)
    rows, cols = w.shape
    cnt = np.zeros(256, dtype=np.uint64)
    _check(lib().orc_histogram(_ptr(w, ctypes.c_uint16), rows, cols,
                               _ptr(cnt, ctypes.c_uint64)), "histogram")
    return cnt


def code_lengths(cnt, lmax: int = 12) -> np.ndarray:
    cnt = np.ascontiguousarray(cnt, dtype=np.uint64)
    assert cnt.shape == (256,)
    out = np.zeros(256, dtype=np.uint8)
    _check(lib().orc_code_lengths(_ptr(cnt, ctypes.c_uint64), lmax,
                                  _ptr(out, ctypes.c_uint8)), "code_lengths")
    return out


def canonical_codes(lengths) -> np.ndarray:
    ln = np.ascontiguousarray(lengths, dtype=np.uint8)
    out = np.zeros(256, dtype=np.uint32)
    _check(lib().orc_canonical_codes(_ptr(ln, ctypes.c_uint8),
                                     _ptr(out, ctypes.c_uint32)), "canonical_codes")
    return out


def blob_size(w: np.ndarray, tile_cols: int = 512, lmax: int = 12,
              tile_rows: int = 8, streams: int = 1) -> int:
    w = np.ascontiguousarray(w, dtype=np.uint16)
    rows, cols = w.shape
    size = ctypes.c_int64()
    if streams == 1:
        rc = lib().orc_blob_size(_ptr(w, ctypes.c_uint16), rows, cols, tile_rows,
                                 tile_cols, lmax, ctypes.byref(size))
    else:
        rc = lib().orc_blob_size_streams(_ptr(w, ctypes.c_uint16), rows, cols, tile_rows,
                                         tile_cols, lmax, streams, ctypes.byref(size))
    _check(rc, "blob_size")
    return size.value


def encode(w: np.ndarray, tile_cols: int = 512, lmax: int = 12,
           tile_rows: int = 8, streams: int = 1) -> np.ndarray:
    """BF16 bit patterns [rows, cols] -> blob (uint8 array); `streams` bit
    streams per lane and tile (1, 2 or 4)."""
    w = np.ascontiguousarray(w, dtype=np.uint16)
    rows, cols = w.shape
    n = blob_size(w, tile_cols, lmax, tile_rows, streams)
    blob = np.zeros(n, dtype=np.uint8)
    size = ctypes.c_int64()
    if streams == 1:
        rc = lib().orc_encode(_ptr(w, ctypes.c_uint16), rows, cols, tile_rows, tile_cols,
                              lmax, _ptr(blob, ctypes.c_uint8), n, ctypes.byref(size))
    else:
        rc = lib().orc_encode_streams(_ptr(w, ctypes.c_uint16), rows, cols, tile_rows,
                                      tile_cols, lmax, streams, _ptr(blob, ctypes.c_uint8), n,
                                      ctypes.byref(size))
    _check(rc, "encode")
    assert size.value == n
    return blob


def blob_info(blob: np.ndarray) -> tuple[int, int]:
    blob = np.ascontiguousarray(blob, dtype=np.uint8)
    rows, cols = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().orc_blob_info(_ptr(blob, ctypes.c_uint8), blob.size,
                               ctypes.byref(rows), ctypes.byref(cols)), "blob_info")
    return rows.value, cols.value


def decode(blob: np.ndarray) -> np.ndarray:
    blob = np.ascontiguousarray(blob, dtype=np.uint8)
    rows, cols = blob_info(blob)
    out = np.zeros((rows, cols), dtype=np.uint16)
    _check(lib().orc_decode(_ptr(blob, ctypes.c_uint8), blob.size,
                            _ptr(out, ctypes.c_uint16), out.size), "decode")
    return out


def decode_tiles(blob: np.ndarray, tile_begin: int, tile_end: int,
                 out: np.ndarray | None = None) -> np.ndarray:
    blob = np.ascontiguousarray(blob, dtype=np.uint8)
    rows, cols = blob_info(blob)
    if out is None:
        out = np.zeros((rows, cols), dtype=np.uint16)
    assert out.dtype == np.uint16 and out.flags.c_contiguous and out.size >= rows * cols
    _check(lib().orc_decode_tiles(_ptr(blob, ctypes.c_uint8), blob.size, tile_begin,
                                  tile_end, _ptr(out, ctypes.c_uint16), out.size),
           "decode_tiles")
    return out


def gemv(w: np.ndarray, x: np.ndarray, row_begin: int = 0,
         row_end: int | None = None) -> np.ndarray:
    """FP64 y[b, n] for n in [row_begin, row_end); W and x are BF16 bit patterns.

    Returns the full [batch, rows] array; rows outside the range are zero."""
    w = np.ascontiguousarray(w, dtype=np.uint16)
    x = np.ascontiguousarray(x, dtype=np.uint16)
    rows, cols = w.shape
    if x.ndim == 1:
        x = x.reshape(1, -1)
    batch = x.shape[0]
    assert x.shape[1] == cols
    row_end = rows if row_end is None else row_end
    y = np.zeros((batch, rows), dtype=np.float64)
    _check(lib().orc_gemv(_ptr(w, ctypes.c_uint16), rows, cols, _ptr(x, ctypes.c_uint16),
                          batch, row_begin, row_end, _ptr(y, ctypes.c_double)), "gemv")
    return y


# ---- variant NWR1: the ranked unary code -----------------------------------

def rank_table(w: np.ndarray, tile_cols: int = 512, ranks: int = 7,
               tile_rows: int = 8) -> list[int]:
    """The values of exponent bits 14..8 that get ranks, in rank order."""
    w = np.ascontiguousarray(w, dtype=np.uint16)
    rows, cols = w.shape
    table = np.zeros(7, dtype=np.uint8)
    n = ctypes.c_int()
    _check(lib().orc_rank_table(_ptr(w, ctypes.c_uint16), rows, cols, tile_rows, tile_cols,
                                ranks, _ptr(table, ctypes.c_uint8), ctypes.byref(n)),
           "rank_table")
    return [int(v) for v in table[:n.value]]


def rank_encode(w: np.ndarray, tile_cols: int = 512, ranks: int = 7,
                tile_rows: int = 8) -> np.ndarray:
    """BF16 bit patterns [rows, cols] -> NWR1 blob (uint8 array)."""
    w = np.ascontiguousarray(w, dtype=np.uint16)
    rows, cols = w.shape
    size = ctypes.c_int64()
    _check(lib().orc_rank_blob_size(_ptr(w, ctypes.c_uint16), rows, cols, tile_rows,
                                    tile_cols, ranks, ctypes.byref(size)), "rank_blob_size")
    blob = np.zeros(size.value, dtype=np.uint8)
    got = ctypes.c_int64()
    _check(lib().orc_rank_encode(_ptr(w, ctypes.c_uint16), rows, cols, tile_rows, tile_cols,
                                 ranks, _ptr(blob, ctypes.c_uint8), blob.size,
                                 ctypes.byref(got)), "rank_encode")
    assert got.value == blob.size
    return blob


def rank_decode(blob: np.ndarray) -> np.ndarray:
    """NWR1 blob -> BF16 bit patterns [rows, cols]."""
    blob = np.ascontiguousarray(blob, dtype=np.uint8)
    if blob.size < 32:
        raise OracleError(ORC_E_CORRUPT, "rank_decode")
    rows = int.from_bytes(blob[16:24].tobytes(), "little")
    cols = int.from_bytes(blob[24:32].tobytes(), "little")
    if not (1 <= rows <= 1 << 32 and 1 <= cols <= 1 << 32) or rows * cols > 1 << 34:
        raise OracleError(ORC_E_CORRUPT, "rank_decode")
    out = np.zeros((rows, cols), dtype=np.uint16)
    _check(lib().orc_rank_decode(_ptr(blob, ctypes.c_uint8), blob.size,
                                 _ptr(out, ctypes.c_uint16), out.size), "rank_decode")
    return out


# ---- variant NWE1: rare exponents in verbatim runs -------------------------

def escape_encode(w: np.ndarray, tile_cols: int = 512, lmax: int = 7, keep: int = 16,
                  tile_rows: int = 8) -> np.ndarray:
    """BF16 bit patterns [rows, cols] -> NWE1 blob (uint8 array): the `keep`
    most frequent exponent bytes coded, runs of 64 holding another one verbatim."""
    w = np.ascontiguousarray(w, dtype=np.uint16)
    rows, cols = w.shape
    size = ctypes.c_int64()
    _check(lib().orc_escape_blob_size(_ptr(w, ctypes.c_uint16), rows, cols, tile_rows,
                                      tile_cols, lmax, keep, ctypes.byref(size)),
           "escape_blob_size")
    blob = np.zeros(size.value, dtype=np.uint8)
    got = ctypes.c_int64()
    _check(lib().orc_escape_encode(_ptr(w, ctypes.c_uint16), rows, cols, tile_rows, tile_cols,
                                   lmax, keep, _ptr(blob, ctypes.c_uint8), blob.size,
                                   ctypes.byref(got)), "escape_encode")
    assert got.value == blob.size
    return blob


def escape_decode(blob: np.ndarray) -> np.ndarray:
    """NWE1 blob -> BF16 bit patterns [rows, cols]."""
    blob = np.ascontiguousarray(blob, dtype=np.uint8)
    if blob.size < 32:
        raise OracleError(ORC_E_CORRUPT, "escape_decode")
    rows = int.from_bytes(blob[16:24].tobytes(), "little")
    cols = int.from_bytes(blob[24:32].tobytes(), "little")
    if not (1 <= rows <= 1 << 32 and 1 <= cols <= 1 << 32) or rows * cols > 1 << 34:
        raise OracleError(ORC_E_CORRUPT, "escape_decode")
    out = np.zeros((rows, cols), dtype=np.uint16)
    _check(lib().orc_escape_decode(_ptr(blob, ctypes.c_uint8), blob.size,
                                   _ptr(out, ctypes.c_uint16), out.size), "escape_decode")
    return out
