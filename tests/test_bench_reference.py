"""The bench's reference arm (the CPU oracle) keeps the JSON-line contract: one line
with the metric, value, unit, impl, the CPU baseline description and an e2e entry
with no host-device traffic; its ms_per_step is time it actually spent (the steps fit
in the run's own wall clock), with the whole-table extrapolation in a field apart."""
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    t0 = time.perf_counter()
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "kaggle",
                          "--steps", "2", "--warmup", "3", "--ref-budget-s", "5"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    wall = time.perf_counter() - t0
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 3
    assert d["ms_per_step"] / 1e3 * (d["steps"] + d["warmup"]) < wall
    assert d["extrapolated_full_step_ms"] > d["ms_per_step"]
    assert abs(d["value"] - d["rows_per_step"] / (d["ms_per_step"] / 1e3)) < 1e-6 * d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
