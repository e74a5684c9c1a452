"""bench.py's reference arm (the fp64 oracle timed on the host cores) without a
GPU: each configuration prints one JSON line with the contract's keys, and a
rank other than 0 prints nothing."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(args, env_extra=None):
    env = dict(os.environ)
    env.setdefault("OMP_NUM_THREADS", "4")
    if env_extra:
        env.update(env_extra)
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True, text=True,
                         env=env, cwd=ROOT, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    return [l for l in out.stdout.splitlines() if l.startswith("{")]


@pytest.mark.parametrize("config", ["ragged", "encoder", "qkv_decode"])
def test_reference_arm_prints_one_contract_line(oracle_lib, config):
    lines = run_bench(["--impl", "reference", "--config", config, "--steps", "1", "--warmup", "1"])
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["value"] > 0 and d["steps"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_reference_arm_other_ranks_stay_silent(oracle_lib):
    assert run_bench(["--impl", "reference", "--steps", "1", "--warmup", "1"],
                     {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}) == []
