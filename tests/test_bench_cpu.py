"""bench.py on the CPU: the reference arm's JSON line (the oracle timed on the
host), and the kernel-code hash that keys the ncu traffic summaries."""
import json
import os
import subprocess
import sys

import pytest

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def run_bench(*args, env=None):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                         capture_output=True, text=True, timeout=600,
                         env={**os.environ, **(env or {})})
    assert out.returncode == 0, out.stderr[-2000:]
    return out.stdout


def test_reference_arm_line():
    line = json.loads(run_bench("--impl", "reference", "--steps", "2", "--warmup", "1")
                      .strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["steps"] == 2 and line["warmup"] == 1
    for key in ("metric", "value", "unit", "n_gpus", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config"):
        assert key in line, key
    assert line["config"]["workload"] == "llama31_8b_stack"
    assert line["value"] > 0 and line["unit"] == "GB/s" and line["higher_is_better"] is True
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_are_silent():
    assert run_bench("--impl", "reference", "--steps", "1", "--warmup", "1",
                     env={"RANK": "1", "WORLD_SIZE": "2"}).strip() == ""


def test_kernel_hash_ignores_comments(tmp_path, monkeypatch):
    code = "int f(int a) {\n  return a + 1;  // add one\n}\n"
    a = tmp_path / "a.cu"
    a.write_text(code)
    b = tmp_path / "b.cu"
    b.write_text("// a header comment\n\n" + code.replace("// add one", "// plus one") + "\n")
    c = tmp_path / "c.cu"
    c.write_text(code.replace("a + 1", "a + 2"))
    hashes = {}
    for p in (a, b, c):
        monkeypatch.setattr(bench, "KERNEL_SOURCE", str(p))
        hashes[p.name] = bench.kernel_source_hash()
    assert hashes["a.cu"] == hashes["b.cu"] != hashes["c.cu"]


def test_traffic_summary_used_only_for_the_kernel_code_it_was_taken_on(tmp_path, monkeypatch):
    """A committed ncu traffic number is reported only while the kernel code
    (comments aside) is the code the capture ran on; otherwise traffic is null."""
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        data = json.load(f)
    current = bench.kernel_source_hash()
    for key, entry in data.items():
        if key.startswith("_"):
            continue
        workload, b = key.split("/b")
        got = bench.profile_traffic(workload, int(b))
        if entry["kernel_sha"] == current:
            assert got == pytest.approx(entry["dram_bytes_per_launch"])
        else:
            assert got is None


def test_traffic_key_names_the_compressed_format():
    """The default format has no suffix; another code or stream count has its own
    key, so a line for one format never reports another format's traffic."""
    import argparse
    ns = lambda **kw: argparse.Namespace(**{"code": "prefix", "streams": 1, **kw})  # noqa: E731
    assert bench.format_suffix(ns()) == ""
    assert bench.format_suffix(ns(code="escape")) == "_escape"
    assert bench.format_suffix(ns(code="rank", streams=1)) == "_rank"
    assert bench.format_suffix(ns(streams=2)) == "_s2"
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        data = json.load(f)
    assert "attn_4096_outliers_escape/b1" in data
    assert data["attn_4096_outliers_escape/b1"]["dram_bytes_per_launch"] != \
        data["attn_4096_outliers/b1"]["dram_bytes_per_launch"]
