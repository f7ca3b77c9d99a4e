"""The C ABI's device calls from a strict-C99 program (tests/c_abi_device.c) on
a GPU: decompression bit-exact, GEMV through both kernels within the parity
tolerance of the FP64 oracle."""
import os
import shutil
import subprocess

import numpy as np
import pytest

from conftest import ROOT
from lossless_bf16_weight_nwc_b200 import synth

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
PKG = os.path.join(ROOT, "lossless_bf16_weight_nwc_b200")
CUDA = "/usr/local/cuda"


def test_c_program_device_calls(tmp_path, orc):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if not shutil.which("gcc"):
        pytest.skip("no C compiler")
    from lossless_bf16_weight_nwc_b200 import build
    lib = build.build()
    exe = str(tmp_path / "c_abi_device")
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                           "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "c_abi_device.c"), lib,
                           f"-L{CUDA}/lib64", "-lcudart", f"-Wl,-rpath,{PKG}",
                           f"-Wl,-rpath,{CUDA}/lib64", "-o", exe])
    prefix = str(tmp_path / "out")
    res = subprocess.run([exe, prefix], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr
    vals = dict(line.split() for line in res.stdout.splitlines())
    i, j = np.meshgrid(np.arange(300), np.arange(1000), indexing="ij")
    w = (0x3C00 + (37 * i + 11 * j) % 1024).astype(np.uint16)
    bi, bj = np.meshgrid(np.arange(40), np.arange(1000), indexing="ij")
    x = (0x3F80 + (bi + 3 * bj) % 64).astype(np.uint16)
    assert np.array_equal(np.fromfile(prefix + ".w", dtype=np.uint16).reshape(300, 1000), w)
    wf = synth.bf16_bits_to_float(w).astype(np.float64)
    for name, batch in (("y1", 3), ("y40", 40)):
        y = np.fromfile(prefix + "." + name, dtype=np.float32).reshape(batch, 300)
        ref = orc.gemv(w, x[:batch])
        xf = synth.bf16_bits_to_float(x[:batch]).astype(np.float64)
        bound = 1e-2 * np.outer(np.linalg.norm(xf, axis=1), np.linalg.norm(wf, axis=1)) * 2.0 ** -8
        assert (np.abs(y - ref) <= bound).all(), name
    assert vals["b3_tensor_cores"] == "0" and vals["b3_launches"] == "1"
    assert vals["b40_tensor_cores"] == "1" and vals["b40_launches"] == "1"
    assert vals["device_error"] == "0" and vals["word"] == "0"
    assert vals["bad_batch"] == "1"                       # NWC_ERR_INVALID_ARG
