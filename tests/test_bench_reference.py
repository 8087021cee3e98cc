"""bench.py's reference arm (the CPU oracle timed on the host cores, on bounded
samples of the workload): one JSON line with the library arm's config keys,
and a ms_per_step that is what each step took, so that steps x ms_per_step
fits inside the run's own clock."""
from __future__ import annotations

import json
import os
import subprocess
import sys
import time

import bench
from quantized_attention_07_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_line_matches_its_own_clock():
    steps, warmup = 2, 3
    t0 = time.perf_counter()
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload",
                        "small_d64", "--steps", str(steps), "--warmup", str(warmup)],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    wall_ms = 1e3 * (time.perf_counter() - t0)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["steps"] == steps
    assert line["value"] > 0 and line["unit"] == "TOPS" and line["higher_is_better"] is True
    # every step, warm-up included, ran inside this process's lifetime
    assert line["ms_per_step"] * (steps + warmup) <= wall_ms
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["value"] == line["value"] and cpu["cores"] >= 1
    assert cpu["projected_ms_per_workload"] > 0
    assert line["e2e"] == {"value": line["value"], "unit": "TOPS", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    # the same config object as the library's arm
    wl = W.WORKLOADS["small_d64"]
    assert line["config"] == bench.config_of(wl, W.make_inputs(wl), 1)
