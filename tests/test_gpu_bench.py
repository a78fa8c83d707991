"""bench.py on the GPU, on a small case of the default workload: one JSON
line with every field of the contract, the device and end-to-end figures
positive and consistent."""

import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_line_small_case():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--cells", "2", "--steps", "5", "--warmup", "3",
           "--no-cpu-baseline"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in d, key
    assert d["value"] > 0 and d["n_gpus"] == 1 and d["steps"] == 5
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["achieved"] > 0 and 0 < r["frac"] < 1.5 and r["unit"] == "GB/s"
    e = d["e2e"]
    assert 0 < e["value"] <= d["value"] * 1.05 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    # cells 0, 1 and the reuse source of any reuse cell among them: fused stored cells, plain reuse decodes
    assert d["gpu_launches"] == 5 * d["config"]["cells_run"]
    assert d["clocks"]["sm_max_mhz"] > 0
