"""The benchmark's contract on the CPU: the reference arm (the fp64 oracle on
the host cores) prints one JSON line with the keys the driver reads, and the
argument rules hold.  The GPU arm is exercised on the B200 only."""
import contextlib
import io
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_reference_arm_json_line():
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3", "--ref-channels", "4"])
    lines = [l for l in buf.getvalue().splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and "4 of 4096 channels" in cb["sample"]
    assert d["config"]["T"] == 65536 and "long" in d["config"]["workload"]


def test_warmup_must_be_at_least_three():
    with pytest.raises(SystemExit):
        bench.main(["--impl", "reference", "--warmup", "2"])


def test_defaults_and_byte_counts():
    a = bench.parse_args([])
    assert a.gpus == 1 and a.warmup >= 3 and a.workload == "long" and a.impl == "ours"
    w = bench.wl.WORKLOADS["long"]
    assert bench.algorithmic_bytes_per_tc(w) == 32
    assert bench.backward_bytes_per_tc(w) == 48
    assert bench.algorithmic_bytes_per_tc(bench.wl.WORKLOADS["lm_layer"]) == 24
    assert bench.backward_bytes_per_tc(bench.wl.WORKLOADS["lm_layer"]) == 36
    assert bench.decode_bytes_per_channel(bench.wl.WORKLOADS["decode"]) == 40


def test_kernel_source_hash_ignores_comments_only(tmp_path, monkeypatch):
    """Recorded DRAM traffic stays attached to the code it measured: editing
    a comment keeps the hash, editing code changes it."""
    src = "// a kernel\n__global__ void k(float *x) { x[0] = 1.f; /* one store */ }\n"
    (tmp_path / "k.cuh").write_text(src)
    monkeypatch.setattr(bench, "CSRC", str(tmp_path))
    h0 = bench.kernel_source_hash()
    (tmp_path / "k.cuh").write_text(src.replace("a kernel", "the kernel").replace("one store", "1 store"))
    assert bench.kernel_source_hash() == h0
    (tmp_path / "k.cuh").write_text(src.replace("1.f", "2.f"))
    assert bench.kernel_source_hash() != h0


def test_recorded_traffic_entries_are_complete():
    """Every entry of the committed traffic record names its kernel, the
    source hash it was taken on, and read + write bytes that add up."""
    with open(bench.TRAFFIC_FILE) as f:
        d = json.load(f)
    assert {"long", "long:backward", "lm_layer", "stiff", "lti", "attention"} <= set(d)
    for e in d.values():
        assert e["kernel"] in (1, 2) and len(e["kernel_sha"]) == 16
        rw = e["dram_read_bytes_per_launch"] + e["dram_write_bytes_per_launch"]
        assert abs(rw - e["dram_bytes_per_launch"]) < 1.0
