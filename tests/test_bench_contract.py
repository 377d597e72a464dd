"""The bench's JSON line on the CPU: the reference arm (the oracle timed on the host cores)
prints one line with the contract's keys, names every workload option in its config, and
only rank 0 prints under a multi-rank launch."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env_extra=None):
    env = dict(os.environ, **(env_extra or {}))
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", *args],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    return [json.loads(line) for line in p.stdout.splitlines() if line.startswith("{")]


@pytest.mark.parametrize("extra,needle", [([], None), (["--rla"], "residual linear attention"),
                                          (["--config", "c3", "--score", "minmax"], "minmax scores"),
                                          (["--config", "c3", "--stats", "bf16"], "bf16 block statistics")])
def test_reference_arm_line(extra, needle):
    args = ["--steps", "2", "--warmup", "1"]
    if "--config" not in extra:
        args += ["--config", "c1"]
    lines = _run(args + extra)
    assert len(lines) == 1
    j = lines[0]
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in j, key
    assert j["impl"] == "reference" and j["steps"] == 2 and j["value"] > 0
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["value"] == j["value"]
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["e2e"]["d2h_bytes_per_step"] == 0
    if needle:
        assert needle in j["config"]["workload"]


def test_reference_arm_prints_on_rank_zero_only():
    assert _run(["--config", "c1", "--steps", "1", "--warmup", "1"], {"RANK": "1", "WORLD_SIZE": "2"}) == []


def test_block_score_option_refuses_index_scored_workloads():
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "c2",
                        "--score", "mean", "--steps", "1", "--warmup", "1"], cwd=ROOT, capture_output=True,
                       text=True, timeout=300)
    assert p.returncode != 0 and "block-scored" in (p.stderr + p.stdout)
