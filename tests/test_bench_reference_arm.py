"""The reference arm of bench.py (the float64 oracle timed on the host cores) on CPU: one JSON line
with the keys every bench line carries, rank 0 only."""
import json
import os
import subprocess
import sys

import bench

ARGS = [sys.executable, os.path.join(bench.ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
        "--warmup", "3"]


def _run(env_extra):
    env = dict(os.environ, **env_extra)
    r = subprocess.run(ARGS, capture_output=True, text=True, timeout=600, env=env, cwd=bench.ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    return [ln for ln in r.stdout.splitlines() if ln.strip()]


def test_reference_line_has_the_contract_keys():
    lines = _run({"RANK": "0", "WORLD_SIZE": "1"})
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "GB/s"
    assert d["higher_is_better"] is True and d["steps"] == 2 and d["warmup"] == 3
    assert d["value"] > 0 and d["config"]["workload"] == "llama7b_mha"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_runs_on_rank_zero_only():
    assert _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}) == []
