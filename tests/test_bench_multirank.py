"""Multi-rank plumbing of bench.py on CPU: two gloo ranks stand in for two GPUs.

The fused path shards into independent replicas (no data exchange), so ranks
only meet for barriers and for the max over ranks of the step times; the
whole-job rate is all ranks' work divided by the slowest rank's time.  The
reference arm runs on rank 0 only; the other ranks return without work.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, os, sys
sys.path.insert(0, os.environ["RFA_ROOT"])
import torch.distributed as dist
import datetime
import bench
rank = int(os.environ["RANK"]); world = int(os.environ["WORLD_SIZE"])
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
bench.barrier(world)
ms = bench.max_over_ranks(1.0 + 2.0 * rank, world)     # rank 0: 1 ms, rank 1: 3 ms
rate = bench.job_throughput(100.0, world, ms)
class A: pass
a = A(); a.workload = "tiny"; a.steps = 1; a.warmup = 0; a.gpus = world
ref = bench.run_reference(a, world, rank) if rank == 1 else None
bench.barrier(world)
dist.destroy_process_group()
print(json.dumps({"rank": rank, "ms": ms, "rate": rate, "ref": ref}))
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_take_the_slowest_time_and_sum_the_work(tmp_path):
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RFA_ROOT=ROOT, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", CHILD], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            o, e = p.communicate(timeout=180)
        except subprocess.TimeoutExpired:
            p.kill()
            pytest.fail("gloo rank did not finish")
        assert p.returncode == 0, e[-2000:]
        outs.append(json.loads(o.strip().splitlines()[-1]))
    for r in outs:
        assert r["ms"] == pytest.approx(3.0)              # max over ranks
        assert r["rate"] == pytest.approx(100.0 * 2 / 3e-3)  # both ranks' units / slowest time
    assert outs[1]["ref"] == 0  # reference arm: non-zero ranks exit 0 without work
