"""bench.py's command-line contract, checked on the CPU through its reference
arm (the FP64 oracle timed on the host cores): one JSON line with the keys
and units the round-end runs read, silence on ranks other than 0, and the
warm-up floor."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args, env=None):
    return subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True, text=True,
                          timeout=300, env=dict(os.environ, **(env or {})))


def test_reference_arm_prints_one_contract_line():
    r = _bench("--impl", "reference", "--steps", "3", "--warmup", "3")
    assert r.returncode == 0, r.stderr
    lines = [x for x in r.stdout.splitlines() if x.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert isinstance(d["metric"], str) and d["metric"]
    assert d["unit"] == "tokens/s" and d["value"] > 0
    assert d["n_gpus"] == 1 and d["warmup"] == 3 and 1 <= d["steps"] <= 3
    assert d["ms_per_step"] > 0
    # value is the throughput of the timed steps: one token per sampled stream per step
    n = d["config"]["streams_per_step"]
    assert n >= 1
    assert abs(d["value"] - n * 1e3 / d["ms_per_step"]) <= 1e-6 * d["value"]
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["vs_baseline"] is None and d["dtype"] == "f64" and d["data"] == "synthetic"
    assert d["config"]["workload"] == "decode_32x32k"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["unit"] == d["unit"]
    assert cb["cores"] >= 1 and isinstance(cb["sample"], str) and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_is_silent_on_other_ranks():
    r = _bench("--impl", "reference", "--steps", "3", "--warmup", "3", env={"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_warmup_floor_is_enforced():
    r = _bench("--impl", "reference", "--steps", "1", "--warmup", "2")
    assert r.returncode != 0
    assert "warmup" in r.stderr
