"""The benchmark's multi-process path on the CPU: world size 2 over gloo.

On one GPU the P ranks of the method are simulated, so several GPUs run independent replicas; the
only collective is the max over ranks of the timings.  These tests run that host logic as two
CPU processes: the real torchrun launch of the reference arm (rank 0 alone prints one JSON line)
and the max-over-ranks reduction.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_reference_arm_under_torchrun_prints_one_line_from_rank0():
    cmd = ["timeout", "-k", "10", "240", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node", "2", "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "pr1", "--gpus", "2",
           "--steps", "2", "--warmup", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


_WORKER = r"""
import datetime, os, sys
sys.path.insert(0, os.environ["HQ_ROOT"])
import torch.distributed as dist
import bench
rank = int(sys.argv[1])
dist.init_process_group("gloo", init_method="tcp://127.0.0.1:" + sys.argv[2], rank=rank, world_size=2,
                        timeout=datetime.timedelta(seconds=60))
v = bench.max_over_ranks(1.5 + rank, 2)
bench.barrier(2)
print("RESULT", rank, v, flush=True)
dist.destroy_process_group()
"""


def test_max_over_ranks_gloo_world2():
    port = str(_free_port())
    env = dict(os.environ, HQ_ROOT=ROOT)
    procs = [subprocess.Popen(["timeout", "-k", "10", "120", sys.executable, "-c", _WORKER, str(r), port],
                              stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True, env=env)
             for r in range(2)]
    outs = [p.communicate() for p in procs]
    for p, (out, err) in zip(procs, outs):
        assert p.returncode == 0, err[-2000:]
    got = sorted(l.split() for o, _ in outs for l in o.splitlines() if l.startswith("RESULT"))
    assert got == [["RESULT", "0", "2.5"], ["RESULT", "1", "2.5"]]
