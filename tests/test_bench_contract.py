"""bench.py's command-line contract, checked on the CPU: the reference arm (the fp64
oracle on the host cores) prints one JSON line with the keys a driver reads, other ranks
of a multi-rank launch exit 0 without work, and forward-only options are rejected on
the fwd+bwd pass."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args, env_extra=None, timeout=300):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=timeout)


def test_reference_arm_prints_one_json_line_with_the_contract_keys():
    r = _bench("--impl", "reference", "--steps", "1", "--warmup", "0")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "p720_pipelined" and d["config"]["pass"] == "fwdbwd"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_without_work():
    r = _bench("--impl", "reference", "--steps", "1", "--warmup", "0", env_extra={"RANK": "1", "WORLD_SIZE": "2"},
               timeout=120)
    assert r.returncode == 0 and not r.stdout.strip()


def test_fp8_is_forward_only_on_the_command_line():
    r = _bench("--fp8", timeout=120)
    assert r.returncode != 0 and "--pass fwd" in r.stderr
