"""bench.py's JSON line on a GPU (the one-token LLM workload, a few steps): one line that
carries every key of the benchmark contract, each consistent with the others."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_line_contract():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "llm_small_m1",
           "--steps", "20", "--warmup", "3", "--attr-steps", "5", "--e2e-steps", "2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-3000:]
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "roofline", "cpu_baseline", "e2e", "gpu_launches", "clocks"):
        assert k in d, k
    assert (d["n_gpus"], d["steps"], d["warmup"]) == (1, 20, 3)
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["unit"] == "TFLOPS"
    assert d["vs_baseline"] is None  # no published figure for this metric and workload
    assert "llm_small_m1" in d["config"]["workload"]
    # value: the step's FLOPs over its time (GFLOP / ms = TFLOP/s)
    assert d["value"] > 0
    assert abs(d["value"] - d["config"]["gflop_per_step_per_gpu"] / d["ms_per_step"]) \
        <= 1e-6 * d["value"]
    # each layer one kernel at one token: two launches per step
    assert d["gpu_launches"] == 2 * d["steps"]
    ro = d["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in ro, k
    assert ro["bound"] == "hbm" and ro["unit"] == "GB/s"
    assert abs(ro["frac"] - ro["achieved"] / ro["peak"]) <= 1e-9
    assert 0 < ro["frac"] < 1.2
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0 and cb["sample"]
    e = d["e2e"]
    assert e["unit"] == d["unit"] and 0 < e["value"] <= d["value"]
    assert e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    c = d["clocks"]
    assert c is not None and c["sm_mhz"] > 0 and c["sm_max_mhz"] > 0
    assert isinstance(c["reasons"], list) and c["samples"] >= 1
