"""bench.py's reference arm on the CPU: the oracle timed on a bounded sample, one JSON line.

The reference arm runs no GPU code; these tests run it on small batches of the E4M3-cache and
verification workloads and check the line's contract fields.
"""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _reference_line(*args):
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0",
           *args]
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, lines
    return json.loads(lines[0])


@pytest.mark.parametrize("args,name_part", [
    (["--workload", "3", "--batch", "1", "--kv-dtype", "e4m3"], "_e4m3"),
    (["--workload", "6", "--batch", "1"], "verify4"),
])
def test_reference_arm_line(args, name_part):
    line = _reference_line(*args)
    assert line["impl"] == "reference"
    assert name_part in line["config"]["workload"]
    assert line["unit"] == "GB/s" and line["value"] > 0 and line["higher_is_better"] is True
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert "cpu" in cb and cb["sample"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_e4m3_option_rejects_a_chunk_workload():
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0",
           "--workload", "5", "--batch", "1", "--kv-dtype", "e4m3"]
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert p.returncode != 0 and "e4m3" in (p.stderr + p.stdout)


def test_gpus_flag_must_match_the_launch():
    # under a launcher that started a different number of processes, --gpus N is refused instead
    # of silently measuring another count of GPUs
    env = dict(os.environ, WORLD_SIZE="2", RANK="0", LOCAL_RANK="0")
    cmd = [sys.executable, "bench.py", "--gpus", "1", "--steps", "1", "--warmup", "0"]
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert p.returncode == 2 and "WORLD_SIZE is 2" in p.stderr, p.stderr[-2000:]
    assert p.stdout.strip() == ""
