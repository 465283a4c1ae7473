"""The benchmark's command-line contract, on the CPU: `bench.py --impl reference`
(the CPU oracle on a bounded sample of the bench workload) prints one JSON line
with the keys the benchmark driver reads, on the same metric and workload as the
GPU arm; under a multi-rank launch only rank 0 prints it."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra, *args):
    env = dict(os.environ, FP8Q_REF_ROWS="2", OMP_NUM_THREADS="2", **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                          capture_output=True, text=True, env=env, timeout=600, cwd=ROOT)


@pytest.fixture(scope="module")
def reference_line():
    r = _run({}, "--impl", "reference", "--steps", "1", "--warmup", "0")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    return json.loads(lines[0])


def test_reference_line_has_the_driver_keys(reference_line):
    d = reference_line
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "e2e",
              "cpu_baseline", "impl"):
        assert k in d, k
    assert d["impl"] == "reference"
    assert d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["steps"] == 1 and d["n_gpus"] == 1
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"],
                        "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert f"2 of 8192 tokens" in cb["sample"]


def test_reference_arm_times_the_gpu_arms_workload(reference_line):
    sys.path.insert(0, ROOT)
    import bench
    assert reference_line["config"] == bench.workload_config(bench.DEFAULT_M, 1)
    assert reference_line["metric"] == bench.METRIC


def test_reference_arm_prints_nothing_on_other_ranks():
    r = _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"},
             "--impl", "reference", "--steps", "1", "--warmup", "0")
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
