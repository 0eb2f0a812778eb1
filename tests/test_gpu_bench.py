"""bench.py on the GPU, small: the JSON line carries every field of the contract.

A short run on the 16K workload with two decode sequences (a few seconds of GPU
work).  Checked: the standard keys, the roofline against the stated peak and
its source, the live clock record, the end-to-end number with its copied bytes,
the launch count, and the per-workload results at the end of the line.
"""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_line_keeps_the_contract():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--headline", "llama2_7b_16k_prefill",
           "--steps", "3", "--warmup", "3", "--decode-steps", "3", "--e2e-steps", "2",
           "--decode-batch", "2", "--no-cpu-baseline", "--no-other-workloads"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "roofline", "e2e", "gpu_launches", "clocks", "decode"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == 3 and d["warmup"] >= 3
    assert d["config"]["workload"] == "llama2_7b_16k_prefill"
    assert d["value"] > 100 and d["unit"] == "TFLOP/s"
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-6
    assert 0.1 < r["frac"] < 1.3
    assert r["peak_source"].split()[0] in ("measured", "fallback")
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] >= 2 * d["steps"]
    assert d["clocks"]["sm_max_mhz"] > 0 and isinstance(d["clocks"]["reasons"], list)
    dec = d["decode"]
    assert dec["unit"] == "GB/s" and dec["value"] > 0
    assert dec["roofline"]["bound"] == "hbm" and 0.1 < dec["roofline"]["frac"] < 1.3
    # the per-workload results close the line, decode last
    assert list(d)[-1] == "decode"
