"""The bench's multi-process path, on the CPU: two ranks over gloo, launched
as separate processes with the environment torchrun gives them (RANK,
WORLD_SIZE, MASTER_ADDR, MASTER_PORT). The path shards into independent
replicas, so its only collectives are the timing barrier and the max over
ranks; these tests run exactly those helpers, and check that the reference
arm under several ranks prints from rank 0 only."""
import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

RANK_SCRIPT = r"""
import datetime, json, os, sys
sys.path.insert(0, os.environ["AE_ROOT"])
import torch.distributed as dist
import bench
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
ms = 100.0 + 7.0 * rank          # the timed region of this rank
dist.barrier()
m = bench.max_over_ranks(ms, dist, device="cpu")
n = bench.sum_over_ranks(100 + rank, dist, device="cpu")   # each rank's kernel launches
dist.barrier()
v = bench.whole_job_value(480.0, world, m, 10)
print(json.dumps({"rank": rank, "max_ms": m, "value": v, "launches": n}), flush=True)
dist.destroy_process_group()
"""


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank: int, world: int, port: int) -> dict:
    env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
               MASTER_PORT=str(port), AE_ROOT=ROOT)
    env.pop("CUDA_VISIBLE_DEVICES", None)
    return env


def test_two_ranks_agree_on_the_slowest_rank_and_the_whole_job_value():
    port = _free_port()
    procs = [subprocess.Popen([sys.executable, "-c", RANK_SCRIPT], env=_env(r, 2, port), cwd=ROOT,
                              stdout=subprocess.PIPE, stderr=subprocess.PIPE) for r in range(2)]
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=180)
        assert p.returncode == 0, err.decode()[-2000:]
        outs.append(json.loads(out.decode().strip().splitlines()[-1]))
    assert sorted(o["rank"] for o in outs) == [0, 1]
    for o in outs:
        assert o["max_ms"] == 107.0  # rank 1's time: the job is as slow as its slowest rank
        assert o["launches"] == 201  # the whole job's launches: 100 + 101
        # two replicas of 480 audio seconds per 10.7 ms step
        assert abs(o["value"] - 2 * 480.0 / (107.0 / 10 / 1e3)) < 1e-6


def test_single_process_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(12.5, None) == 12.5
    assert bench.sum_over_ranks(7, None) == 7
    assert abs(bench.whole_job_value(480.0, 1, 95.0, 10) - 480.0 / 9.5e-3) < 1e-6


def test_reference_arm_prints_from_rank_zero_only():
    port = _free_port()
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--workload", "frontend", "--steps", "1"]
    quiet = subprocess.run(cmd, env=_env(1, 2, port), cwd=ROOT, capture_output=True, timeout=300)
    assert quiet.returncode == 0 and quiet.stdout.strip() == b""
    loud = subprocess.run(cmd, env=_env(0, 2, port), cwd=ROOT, capture_output=True, timeout=300)
    assert loud.returncode == 0, loud.stderr.decode()[-2000:]
    line = json.loads(loud.stdout.decode().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
