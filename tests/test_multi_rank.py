"""The N > 1 bench plumbing on CPU: two gloo ranks on 127.0.0.1 (no GPU)."""
import json
import os
import socket
import subprocess
import sys
from pathlib import Path

ROOT = Path(__file__).resolve().parents[1]

CHILD = r"""
import os, sys, json
sys.path.insert(0, os.environ["QMM_ROOT"])
import torch.distributed as dist
import bench
dist.init_process_group("gloo")
world, rank = dist.get_world_size(), dist.get_rank()
# each rank took a different time; the job's time is the slowest rank's
t = bench.max_over_ranks(world, 10.0 + 5.0 * rank)
bench.barrier(world)
rate = bench.whole_job_rate(world, 4, 1000, t)
print(json.dumps({"rank": rank, "world": world, "t": t, "rate": rate}), flush=True)
bench.dist_teardown(world)
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port):
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
               LOCAL_RANK=str(rank), WORLD_SIZE=str(world), QMM_ROOT=str(ROOT),
               CUDA_VISIBLE_DEVICES="")
    return env


def test_max_over_ranks_and_job_rate_two_gloo_ranks():
    port = _free_port()
    procs = [subprocess.Popen([sys.executable, "-c", CHILD], env=_env(r, 2, port),
                              stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
             for r in range(2)]
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=180)
        assert p.returncode == 0, err
        outs.append(json.loads(out.strip().splitlines()[-1]))
    for o in outs:
        assert o["world"] == 2
        assert o["t"] == 15.0  # max over ranks, seen identically by both
        # 2 ranks x 4 steps x 1000 units in 15 ms
        assert abs(o["rate"] - 2 * 4 * 1000 / 0.015) < 1e-6


def test_reference_arm_under_torchrun_prints_one_line():
    port = _free_port()
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), str(ROOT / "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "3", "--warmup", "3"]
    r = subprocess.run(cmd, env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["value"] > 0
