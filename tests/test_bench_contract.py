"""bench.py's reference arm on the CPU: the JSON line it prints keeps the contract.

The reference arm times the fp64 oracle on the host cores (there is no installable
reference implementation: the reference is a set of pages).  Here it runs on the
tiny workload with each step's oracle time capped, and the line must carry the
keys, types and values the driver reads, with the same `config` as the GPU arm.
"""
import json
import os
import sys
from types import SimpleNamespace

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from yarn_position_scaling_b200 import synth  # noqa: E402


def test_reference_arm_line(monkeypatch):
    real = bench.oracle_sample
    monkeypatch.setattr(bench, "oracle_sample",
                        lambda w, seconds, seed=0: real(w, min(seconds, 0.2), seed))
    args = SimpleNamespace(headline=synth.TINY.name, steps=2, warmup=1)
    line = bench.reference_arm(args, SimpleNamespace(rank=0))
    json.dumps(line)  # serialisable as one line
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e", "gpu_launches"):
        assert key in line, key
    assert line["value"] > 0 and line["unit"] == "TFLOP/s" and line["higher_is_better"] is True
    assert line["steps"] == 2 and line["warmup"] == 1 and line["n_gpus"] == 1
    assert line["dtype"] == "f64" and line["vs_baseline"] is None and line["gpu_launches"] == 0
    assert line["config"] == bench.workload_config(synth.TINY, 1)
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert cb["unit"] == line["unit"] and "query rows" in cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_do_no_work(monkeypatch):
    monkeypatch.setattr(bench, "oracle_sample", lambda *a, **k: (_ for _ in ()).throw(
        AssertionError("rank != 0 must not run the oracle")))
    args = SimpleNamespace(headline=synth.TINY.name, steps=2, warmup=1)
    assert bench.reference_arm(args, SimpleNamespace(rank=1)) is None
