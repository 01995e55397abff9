"""bench.py's reference arm (the fp64 oracle timed on the host cores) runs end to end on CPU
and prints the JSON line the driver reads; on ranks other than 0 it prints nothing."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(config, env_extra=None, gpus=1):
    env = dict(os.environ, **(env_extra or {}))
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0",
                           "--config", config, "--gpus", str(gpus)], cwd=ROOT, env=env, capture_output=True,
                          text=True, timeout=600)


@pytest.mark.parametrize("config", ["qwen3_1p7b_gqa_b32", "mla_576_512_b16", "cont_batch_b256"])
def test_reference_arm_prints_its_line(config):
    r = _run(config)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["dtype"] == "f64"
    assert d["config"]["workload"] == config
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_is_silent_on_other_ranks():
    r = _run("qwen3_1p7b_gqa_b32", {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}, gpus=2)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_gpus_must_match_the_launched_processes():
    # --gpus 2 in a single process (no torchrun) is refused instead of silently running one GPU
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, "bench.py", "--gpus", "2", "--steps", "1", "--warmup", "0"], cwd=ROOT,
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode != 0 and "torchrun" in r.stderr
