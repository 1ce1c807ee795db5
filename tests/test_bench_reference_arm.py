"""bench.py's reference arm (the fp64 oracle timed on the host cores) prints one JSON line with
the keys the benchmark contract needs; ranks other than 0 print nothing.  CPU only."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra, workload=None):
    env = dict(os.environ, **env_extra)
    extra = ["--workload", workload] if workload else []
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"] + extra, capture_output=True, text=True, env=env, cwd=ROOT, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    return out.stdout


@pytest.mark.parametrize("workload", [None, "decode", "decode_fp8", "fp8", "d256"])
def test_reference_arm_line(workload):
    lines = [l for l in _run({}, workload).splitlines() if l.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in rec, key
    assert rec["impl"] == "reference" and rec["unit"] == "TFLOP/s" and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["cores"] >= 1
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["e2e"]["value"] == rec["value"]


def test_reference_arm_only_rank0_prints():
    assert _run({"RANK": "1", "WORLD_SIZE": "2"}).strip() == ""
