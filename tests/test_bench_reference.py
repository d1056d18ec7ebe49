"""bench.py's reference arm on the CPU: it times the fp64 oracle on a bounded sample and
prints one JSON line carrying every key the benchmark contract asks for (no GPU needed)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


@pytest.mark.parametrize("workload, extra", [
    (3, ["--users", "2", "--length", "48", "--n-items", "5000"]),
    (4, ["--users", "8", "--length", "1500", "--n-items", "5000"]),  # L ~ U{1000 .. 1500}
])
def test_reference_arm_prints_contract_line(workload, extra):
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--workload", str(workload), "--steps", "2",
           "--warmup", "3"] + extra
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert KEYS <= set(j)
    assert j["impl"] == "reference" and j["value"] > 0 and j["higher_is_better"] is True
    assert j["steps"] == 2 and j["warmup"] == 3 and j["n_gpus"] == 1
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["cores"] >= 1
    assert j["e2e"]["value"] == j["value"] and j["e2e"]["h2d_bytes_per_step"] == 0
    assert "weights" not in j["config"]
