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
