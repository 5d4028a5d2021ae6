"""The multi-GPU bench path on the CPU: two gloo ranks run bench.py's rank logic.

`bench.py --gpus N` runs N independent replicas (the decode path has no exchange step): every
rank times the same workload, the whole-job rate divides all ranks' bytes by the slowest rank's
time, and rank 0 alone prints. These tests run that logic with world size 2 over gloo on the
CPU; no GPU and no kernel is involved.
"""

import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r'''
import json, os, sys
import torch
import torch.distributed as dist
sys.path.insert(0, os.environ["FD_ROOT"])
import bench
rank = int(os.environ["RANK"]); world = int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", rank=rank, world_size=world)
dev = torch.device("cpu")
local_ms = [100.0, 250.0][rank]               # the second rank is the slowest
ms_max = bench.max_over_ranks(local_ms, world, dev)
rate = bench.whole_job_gbs(2_000_000_000, 10, world, ms_max)
bench.emit({"rank": rank, "ms_max": ms_max, "value": rate}, rank)
dist.barrier()
dist.destroy_process_group()
'''


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run_ranks(code, world=2, timeout=120):
    port = _free_port()
    procs = []
    for rank in range(world):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), FD_ROOT=ROOT)
        procs.append(subprocess.Popen([sys.executable, "-c", code], env=env, cwd=ROOT,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            out, err = p.communicate(timeout=timeout)
        except subprocess.TimeoutExpired:
            p.kill()
            out, err = p.communicate()
        outs.append((p.returncode, out, err))
    return outs


def test_two_gloo_ranks_take_the_slowest_time_and_rank0_prints():
    outs = _run_ranks(WORKER)
    for rc, out, err in outs:
        assert rc == 0, err[-2000:]
    lines0 = [l for l in outs[0][1].splitlines() if l.strip()]
    lines1 = [l for l in outs[1][1].splitlines() if l.strip()]
    assert len(lines0) == 1 and lines1 == [], (lines0, lines1)
    line = json.loads(lines0[0])
    assert line["ms_max"] == 250.0                       # max over ranks, not rank 0's own time
    # two replicas x 2 GB x 10 steps over 0.25 s
    assert line["value"] == pytest.approx(2 * 2e9 * 10 / 0.25 / 1e9)


def test_reference_arm_ranks_other_than_zero_exit_quietly():
    # under torchrun the oracle arm runs on rank 0 only; rank 1 returns at once with no output
    code = r'''
import os, sys
sys.path.insert(0, os.environ["FD_ROOT"])
sys.argv = ["bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"]
import bench
args = bench.parse_args()
sys.exit(bench.run_reference(args, int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])))
'''
    port = _free_port()
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
               MASTER_PORT=str(port), FD_ROOT=ROOT)
    p = subprocess.run([sys.executable, "-c", code], env=env, cwd=ROOT, capture_output=True,
                       text=True, timeout=120)
    assert p.returncode == 0, p.stderr[-2000:]
    assert p.stdout.strip() == ""


def test_single_rank_helpers():
    import torch
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.whole_job_gbs(10**9, 4, 1, 1000.0) == pytest.approx(4.0)
