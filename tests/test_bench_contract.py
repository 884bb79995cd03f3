"""The bench's JSON contract on the CPU: the reference arm (the oracle on the
host cores) prints one line with every required key, the metric, unit and
config of the measured arm, and only rank 0 prints under a multi-rank launch."""
import json
import os
import subprocess
import sys

import pytest

import bench
from recurrent_state_quantization_lq_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None):
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "LOCAL_WORLD_SIZE"):
        env.pop(k, None)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_line():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert (d["metric"], d["unit"], d["higher_is_better"]) == (bench.METRIC, bench.UNIT, True)
    assert (d["n_gpus"], d["steps"], d["warmup"]) == (1, 1, 3)
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["vs_baseline"] is None
    assert d["data"] == "synthetic" and d["scaling"] == "weak"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["unit"] == d["unit"]
    assert cb["sample"]
    e = d["e2e"]
    assert (e["value"], e["unit"], e["h2d_bytes_per_step"], e["d2h_bytes_per_step"]) == (d["value"], d["unit"], 0, 0)
    assert d["config"]["workload"] == "gdn_b64_h32_d128_w64"      # the default: 64 x 32 heads, d 128, W 64
    wl = inputs.WORKLOADS[d["config"]["workload"]]
    assert d["config"] == bench.bench_config(wl, d["config"]["layers_rotated"], 1)


def test_reference_arm_prints_on_rank_zero_only():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "3"],
             {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1", "LOCAL_WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    assert not [l for l in r.stdout.splitlines() if l.startswith("{")]


@pytest.mark.parametrize("warmup", ["0", "2"])
def test_too_few_warmup_steps_refused(warmup):
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", warmup])
    assert r.returncode != 0
    assert "--warmup must be >= 3" in r.stderr
