"""The benchmark's JSON line on a GPU: one short run of `bench.py` (the hot-path step on
the full 16384-row workload, a few timed steps) must print exactly one line with the keys
and units the measurement contract fixes, consistent with each other."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
def test_bench_line_keys_and_consistency(cuda_device):
    steps, warmup = 5, 3
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--steps", str(steps), "--warmup",
                          str(warmup), "--no-cpu-baseline"], cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    b = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert k in b, k
    assert b["n_gpus"] == 1 and b["steps"] == steps and b["warmup"] == warmup
    assert b["higher_is_better"] is True and b["scaling"] == "weak" and b["unit"] == "GB/s"
    assert b["data"] == "synthetic" and "workload" in b["config"] and "l2" in b["config"]
    # value: algorithmic bytes of the step over the step time
    assert b["value"] > 0 and b["ms_per_step"] > 0
    r = b["roofline"]
    assert r["bound"] in ("tensor", "hbm") and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-3
    assert 0.05 < r["frac"] < 1.5
    e = b["e2e"]
    assert e["unit"] == b["unit"] and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert 0 < e["value"] < b["value"]          # host copies inside the timed region
    assert b["gpu_launches"] == 4 * steps       # the step's four library kernels
    c = b["clocks"]
    assert c["sm_max_mhz"] and c["sm_mhz"] and c["samples"] >= 1
