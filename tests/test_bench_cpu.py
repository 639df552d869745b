"""bench.py's CPU-side contract: the reference arm (the fp64 oracle timed on host cores) and the
bounded CPU baseline. Neither needs a GPU."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config")


def _run(args, env_extra=None, timeout=300):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                          env=env, capture_output=True, text=True, timeout=timeout)


def test_reference_arm_prints_one_contract_line():
    p = _run(["--impl", "reference", "--workload", "small", "--steps", "2", "--warmup", "0",
              "--reference-tokens", "16"])
    assert p.returncode == 0, p.stderr
    lines = [ln for ln in p.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in KEYS:
        assert k in d, k
    assert d["impl"] == "reference"
    assert d["value"] > 0 and d["steps"] == 2 and d["warmup"] >= 3  # the warm-up floor holds
    assert d["higher_is_better"] is True and d["dtype"] == "f64"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    p = _run(["--impl", "reference", "--workload", "small", "--steps", "1",
              "--reference-tokens", "16"], env_extra={"RANK": "1", "WORLD_SIZE": "2"})
    assert p.returncode == 0, p.stderr
    assert p.stdout.strip() == ""


def test_cpu_baseline_is_bounded_and_reports_its_sample():
    sys.path.insert(0, ROOT)
    import bench
    from mhc_hyper_connection_02_b200 import inputs
    w = inputs.small()
    r = bench.cpu_baseline(w, budget_s=0.5, max_passes=5)
    assert r["kind"] == "oracle" and r["value"] > 0 and r["cores"] >= 1
    assert r["unit"] == bench.UNIT
    assert "of 64 tokens" in r["sample"] and "pass" in r["sample"]
