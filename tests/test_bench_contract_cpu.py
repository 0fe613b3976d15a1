"""The benchmark's command-line contract, checked on the CPU: the reference arm (the oracle on
host cores) prints one JSON line with the contract's keys, only rank 0 prints under several
ranks, too few warm-up steps are refused, and the product arm fails loudly (no JSON line) on a
machine without a GPU instead of falling back to the CPU."""
import json
import os
import subprocess
import sys
from pathlib import Path

import pytest
import torch

ROOT = Path(__file__).resolve().parents[1]
FAST_REF = ["--ref-step-budget", "0.3", "--ref-total-budget", "2"]


def run_bench(args, env_extra=None, timeout=300):
    env = dict(os.environ)
    for key in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(key, None)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, str(ROOT / "bench.py"), *args], cwd=ROOT, env=env,
                          capture_output=True, text=True, timeout=timeout)


def json_lines(stdout):
    out = []
    for line in stdout.splitlines():
        line = line.strip()
        if line.startswith("{"):
            out.append(json.loads(line))
    return out


def test_reference_arm_prints_the_contract_line():
    res = run_bench(["--impl", "reference", "--steps", "2", "--warmup", "3", *FAST_REF])
    assert res.returncode == 0, res.stderr
    lines = json_lines(res.stdout)
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference" and d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 3
    for key in ("metric", "unit", "ms_per_step", "higher_is_better", "scaling", "dtype", "data"):
        assert key in d, key
    assert d["value"] > 0 and d["vs_baseline"] is None
    assert isinstance(d["config"]["workload"], str) and d["config"]["workload"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_prints_on_rank_zero_only():
    res = run_bench(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", *FAST_REF],
                    env_extra={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert res.returncode == 0, res.stderr
    assert json_lines(res.stdout) == []
    # the launcher gives every rank one OpenMP thread; rank 0, working alone, takes every core
    res = run_bench(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", *FAST_REF],
                    env_extra={"RANK": "0", "WORLD_SIZE": "2", "LOCAL_RANK": "0", "OMP_NUM_THREADS": "1"})
    assert res.returncode == 0, res.stderr
    lines = json_lines(res.stdout)
    assert len(lines) == 1 and lines[0]["n_gpus"] == 2
    assert lines[0]["cpu_baseline"]["cores"] == len(os.sched_getaffinity(0))


def test_fewer_than_three_warmup_steps_are_refused():
    res = run_bench(["--impl", "reference", "--steps", "1", "--warmup", "2", *FAST_REF])
    assert res.returncode == 2
    assert json_lines(res.stdout) == []


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour on a machine without a GPU")
def test_product_arm_fails_loudly_without_a_gpu():
    res = run_bench(["--steps", "1", "--warmup", "3", "--no-e2e", "--no-cpu-baseline", "--no-workload-set"])
    assert res.returncode != 0
    assert all("value" not in d for d in json_lines(res.stdout))
