"""The benchmark's reference arm (`bench.py --impl reference`): the oracle
timed on the host cores.  Runs on the CPU on the smallest workload and checks
the one JSON line against the benchmark contract: the same metric, unit and
workload name as the GPU arm, the reference marker, a CPU-baseline record and
an end-to-end record without host-device traffic."""
import contextlib
import io
import json
import types

import bench
from weight_only_quantized_g64_b200 import synth


def _run(wl, rank=0, world=1):
    args = types.SimpleNamespace(steps=2, warmup=1)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.reference_arm(args, wl, rank, world)
    return buf.getvalue()


def test_reference_arm_line():
    wl = synth.WORKLOADS[1]
    lines = [ln for ln in _run(wl).splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC
    assert line["unit"] == "GB/s" and line["higher_is_better"] is True
    assert line["value"] > 0 and line["steps"] == 2 and line["warmup"] == 1
    assert line["config"]["workload"] == wl.name
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_print_nothing():
    assert _run(synth.WORKLOADS[1], rank=1, world=2) == ""
