"""bench.py's reference arm (the oracle timed on the host cores) on CPU: the JSON
line it prints carries every key the benchmark contract asks for, and under a
multi-rank launch only rank 0 prints."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BENCH = os.path.join(ROOT, "bench.py")


def _run(extra_env=None, args=()):
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    env.update(extra_env or {})
    cmd = [sys.executable, BENCH, "--impl", "reference", "--workload", "toy_fp32",
           "--steps", "2", "--warmup", "1", *args]
    return subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_line_has_the_contract_keys():
    import bench
    r = _run()
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == "tokens/s"
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 1
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["vs_baseline"] is None and d["data"] == "synthetic"
    assert d["config"]["workload"] == "toy_fp32"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert cb["unit"] == "tokens/s" and "tokens" in cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_config_matches_the_gpu_arm():
    import bench
    import synth
    wl = synth.WORKLOADS["toy_fp32"]
    r = _run()
    d = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][0])
    assert d["config"] == bench.workload_config(wl, 1)


@pytest.mark.parametrize("rank", ["1", "3"])
def test_reference_arm_other_ranks_exit_without_output(rank):
    r = _run({"RANK": rank, "WORLD_SIZE": "4", "LOCAL_RANK": rank}, ("--gpus", "4"))
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
