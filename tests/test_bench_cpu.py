"""bench.py's reference arm (the oracle on the host cores) on the CPU: the
JSON line keeps the benchmark contract, times exactly --steps steps, and
ranks other than 0 exit without work."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None, timeout=300):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          timeout=timeout, env=env, cwd=ROOT)


def _check_line(d, steps, warmup, workload):
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference"
    assert d["steps"] == steps and d["warmup"] == warmup
    assert d["unit"] == "GB/s" and d["higher_is_better"] is True and d["value"] > 0
    assert d["config"]["workload"] == workload
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_tiny():
    r = _run(["--impl", "reference", "--steps", "3", "--warmup", "1", "--config", "tiny"])
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    _check_line(json.loads(lines[0]), 3, 1, "tiny:tiny_256x512:B1")


def test_reference_arm_default_workload_is_bounded():
    """The default workload (4096 x 4096, batch 1) on a row sample sized to
    about --cpu-seconds of oracle work, scaled to the whole layer."""
    r = _run(["--impl", "reference", "--steps", "2", "--warmup", "1", "--cpu-seconds", "0.5"], timeout=120)
    assert r.returncode == 0, r.stderr
    d = json.loads(r.stdout.strip().splitlines()[-1])
    _check_line(d, 2, 1, "llama7b_layer:l7b_4096x4096:B1")
    assert d["config"]["N"] == 4096 and d["config"]["K"] == 4096


def test_reference_arm_other_ranks_exit_quietly():
    r = _run(["--impl", "reference", "--steps", "2", "--warmup", "1", "--config", "tiny"],
             env_extra={"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
