"""Lossless BF16 weight compression with a fused decode-GEMV for B200 (sm_100a).

The product is the C-ABI library libnwc.so (include/nwc.h); `_lib` binds it
with ctypes (loaded on first use, and it raises if the library is missing).
`synth` generates the seeded synthetic inputs; `autotune` picks a matrix's
tile width and code limit by timing the library's GEMV on the device;
`sharded` splits a matrix by output rows over a process group.
"""
import importlib

__all__ = ["CompressedMatrix", "lib"]


def __getattr__(name):
    if name == "lib":
        return importlib.import_module(__name__ + "._lib")
    if name == "CompressedMatrix":
        return importlib.import_module(__name__ + "._lib").CompressedMatrix
    raise AttributeError(name)
