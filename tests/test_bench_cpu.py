"""The benchmark's reference arm (the CPU oracle timed on the host cores) and
its output contract, run here on the CPU: one JSON line from rank 0 with the
keys the benchmark promises, nothing from the other ranks."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

KEYS = ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e")


def _run(env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "1",
                           "--warmup", "3"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)


def test_reference_arm_prints_one_contract_line():
    r = _run({})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    for k in KEYS:
        assert k in d, k
    assert d["impl"] == "reference" and d["unit"] == "TOPS" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["steps"] == 1 and d["data"] == "synthetic"
    assert d["config"]["workload"] == "tiny" and (d["config"]["M"], d["config"]["K"], d["config"]["N"]) == (64, 256, 256)
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    # ms per step restates the metric: 2 M N K operations at `value` TOPS
    assert abs(d["ms_per_step"] - 2.0 * 64 * 256 * 256 / (d["value"] * 1e12) * 1e3) <= 1e-9 + 1e-9 * d["ms_per_step"]


def test_reference_arm_is_silent_on_other_ranks():
    r = _run({"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert not [ln for ln in r.stdout.splitlines() if ln.startswith("{")]


def test_fewer_than_three_warmup_steps_are_refused():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "1",
                        "--warmup", "2"], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "warmup" in (r.stdout + r.stderr)


def test_reference_arm_of_the_sweep_says_unavailable():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--sweep", "--steps", "1", "--warmup", "3"],
                       cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(ln) for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1 and lines[0]["impl"] == "reference" and lines[0]["unavailable"]


def test_reference_arm_of_the_w4a8_variant():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--variant", "w4a8", "--workload", "m256_down",
                        "--steps", "1", "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    d = [json.loads(ln) for ln in r.stdout.splitlines() if ln.startswith("{")][0]
    assert d["impl"] == "reference" and d["value"] > 0 and "int8" in d["dtype"]
    assert d["config"]["workload"] == "m256_down"
