"""The C ABI from C: tests/c_abi_host.c compiles as strict C99 against
include/nwc.h, links libnwc.so, and its host-only calls give the oracle's
blobs and the documented statuses (no GPU)."""
import os
import shutil
import subprocess

import numpy as np
import pytest

from conftest import ROOT

PKG = os.path.join(ROOT, "lossless_bf16_weight_nwc_b200")


@pytest.fixture(scope="module")
def c_program(tmp_path_factory):
    if not shutil.which("gcc"):
        pytest.skip("no C compiler")
    from lossless_bf16_weight_nwc_b200 import build
    lib = build.build()
    out = tmp_path_factory.mktemp("cabi")
    exe = str(out / "c_abi_host")
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                           "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "c_abi_host.c"), lib,
                           f"-Wl,-rpath,{PKG}", "-o", exe])
    return exe, out


def test_c_caller_matches_oracle(c_program, orc):
    exe, out = c_program
    prefix = str(out / "m")
    res = subprocess.run([exe, prefix], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stderr
    vals = dict(line.split() for line in res.stdout.splitlines())
    i, j = np.meshgrid(np.arange(24), np.arange(200), indexing="ij")
    w = (0x3C00 + (37 * i + 11 * j) % 1024).astype(np.uint16)
    nwb1 = np.fromfile(prefix + ".nwb1", dtype=np.uint8)
    nwr1 = np.fromfile(prefix + ".nwr1", dtype=np.uint8)
    assert np.array_equal(nwb1, orc.encode(w, lmax=7))
    assert np.array_equal(nwr1, orc.rank_encode(w, tile_cols=64, ranks=3))
    nwe1 = np.fromfile(prefix + ".nwe1", dtype=np.uint8)
    assert np.array_equal(nwe1, orc.escape_encode(w, tile_cols=128, lmax=7, keep=4))
    assert int.from_bytes(nwe1[104:112].tobytes(), "little") > 0      # some runs verbatim
    assert int(vals["nwe1_device_bytes"]) > nwe1.size + 65536         # blob, table, schedules
    assert int(vals["nwb1_device_bytes"]) == int(vals["blob_device_bytes"]) > nwb1.size
    assert int(vals["schedule_tiles"]) == 3 and int(vals["schedule_ctas"]) == 3
    assert int(vals["corrupt_status"]) == 4          # NWC_ERR_CORRUPT
    assert int(vals["nwr1_device_bytes"]) > nwr1.size    # blob, rank table, schedules, scratch
    assert int(vals["null_matrix_status"]) == 1      # NWC_ERR_INVALID_ARG
    assert int(vals["version"]) > 0
