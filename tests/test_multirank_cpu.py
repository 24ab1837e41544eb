"""The bench's multi-process path, on the CPU: two ranks over gloo, launched
as separate processes with the environment torchrun gives them (RANK,
WORLD_SIZE, MASTER_ADDR, MASTER_PORT). The path shards into independent
clips: each rank takes the clips ae_partition_clips assigns it from a global
batch (greedy token balance, computed on every rank from the lengths alone),
so the only collectives are the timing barrier and the max over ranks. These
tests run those helpers, the partition across two ranks (the oracle on a
tiny model stands in for each rank's device call, which needs a GPU), and
check that the reference arm under several ranks prints from rank 0 only."""
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


PARTITION_SCRIPT = r"""
import datetime, json, os, sys
sys.path.insert(0, os.environ["AE_ROOT"])
import numpy as np
import torch.distributed as dist
import bench, synth
import log_mel_front_b200 as ae
from oracle import oracle as O
rank, world = int(os.environ["RANK"]), int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
lens = [16000, 161, 100, 40000, 5000, 72825, 321, 24000, 3300]
mine = bench.rank_clips(lens, world, rank, ae.ae_partition_clips)
shape = dict(synth.MODEL_SHAPE, hidden=32, heads=2, ffn=48, out_dim=40, embed_dim=24)
W = synth.model_weights("pr1", n_layers=1, shape=shape)
W["stem"]["in_proj"] = (0.02 * np.random.default_rng(11).standard_normal((32, 1024))).astype(np.float32)
clips = synth.global_waves("ragged", lens, mine)
outs = O.encode(clips, W) if clips else []   # this rank's packed batch
got = [None] * world
dist.all_gather_object(got, {"rank": rank, "clips": mine, "rows": [o.tolist() for o in outs],
                             "tokens": sum(ae.ae_num_tokens(lens[i]) for i in mine)})
if rank == 0:
    owner = {}
    for g in got:
        for i in g["clips"]:
            assert i not in owner, "clip on two ranks"
            owner[i] = g
    assert sorted(owner) == list(range(len(lens))), "a clip on no rank"
    toks = [g["tokens"] for g in got]
    assert max(toks) - min(toks) <= max(ae.ae_num_tokens(n) for n in lens), toks
    # the ranks' rows, put back in global clip order, equal the single-rank result
    single = O.encode(synth.global_waves("ragged", lens, list(range(len(lens)))), W)
    for i in range(len(lens)):
        g = owner[i]
        rows = np.array(g["rows"][g["clips"].index(i)]).reshape(-1, 24)
        assert rows.shape == single[i].shape
        assert np.allclose(rows, single[i], rtol=0, atol=1e-12), i
m = bench.max_over_ranks(1.0 + rank, dist, device="cpu")
dist.barrier()
print(json.dumps({"rank": rank, "clips": mine, "max_ms": m}), flush=True)
dist.destroy_process_group()
"""


def test_two_ranks_split_a_batch_and_rejoin_it():
    port = _free_port()
    procs = [subprocess.Popen([sys.executable, "-c", PARTITION_SCRIPT], env=_env(r, 2, port), cwd=ROOT,
                              stdout=subprocess.PIPE, stderr=subprocess.PIPE) for r in range(2)]
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=300)
        assert p.returncode == 0, err.decode()[-3000:]
        outs.append(json.loads(out.decode().strip().splitlines()[-1]))
    a, b = sorted(outs, key=lambda o: o["rank"])
    assert a["clips"] and b["clips"] and not set(a["clips"]) & set(b["clips"])
    assert a["max_ms"] == b["max_ms"] == 2.0


def test_partition_properties():
    """ae_partition_clips (host only): every clip on exactly one part, the parts'
    token totals within one clip of each other, deterministic, one part = all,
    and the bench's per-rank lists follow it."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    import log_mel_front_b200 as ae
    import synth
    rng = np.random.default_rng(8)
    for n_clips, parts in ((1, 1), (7, 3), (256, 8), (300, 7), (5, 8)):
        lens = rng.integers(0, 600000, size=n_clips)
        off = np.concatenate([[0], np.cumsum(lens)])
        part, tok = ae.ae_partition_clips(off, parts)
        assert part.shape == (n_clips,) and part.min() >= 0 and part.max() < parts
        per = [int(ae.ae_num_tokens(int(n))) for n in lens]
        assert list(tok) == [sum(t for t, p in zip(per, part) if p == k) for k in range(parts)]
        assert tok.max() - tok.min() <= max(per)
        assert np.array_equal(ae.ae_partition_clips(off, parts)[0], part)
        got = sorted(i for r in range(parts) for i in bench.rank_clips(list(lens), parts, r, ae.ae_partition_clips))
        assert got == list(range(n_clips))
    lens = synth.clip_lengths("ragged")
    off = np.concatenate([[0], np.cumsum(lens)])
    assert np.all(ae.ae_partition_clips(off, 1)[0] == 0)
    _, tok = ae.ae_partition_clips(off, 8)
    assert tok.max() - tok.min() <= 750
