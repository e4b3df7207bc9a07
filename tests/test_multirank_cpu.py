"""The benchmark's multi-rank plumbing on CPU: two gloo ranks on 127.0.0.1.

With N GPUs the benchmark runs N independent replicas of the stack (one per rank, each
with its own input stream); the only collectives are a barrier around the timed region
and the max over ranks of the measured time.  These tests run that host logic with the
gloo backend and world size 2, and the reference arm under torchrun, where rank 0 alone
runs and prints."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


_WORKER = r"""
import os, sys
sys.path.insert(0, {root!r})
import bench
world, rank, local = bench.dist_setup()
assert (world, rank) == (2, int(os.environ["RANK"]))
bench.dist_barrier(world)
m = bench.dist_max(1.5 + rank, world)
rate = bench.whole_job_rate(world, steps=8, batch=1, ms_max=m)
import torch.distributed as dist
dist.destroy_process_group()
print(f"RESULT {{rank}} {{m}} {{rate}}")
"""


def test_dist_max_and_barrier_two_gloo_ranks():
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", _WORKER.format(root=ROOT)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=240)
        assert p.returncode == 0, err[-2000:]
        outs.append([l for l in out.splitlines() if l.startswith("RESULT")][0].split())
    for _, rank, m, rate in outs:
        # the max over ranks is 2.5 on both; the job rate counts the tokens of both replicas
        assert float(m) == 2.5
        assert abs(float(rate) - 2 * 8 * 1 / 2.5e-3) < 1e-6


@pytest.mark.slow
def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
           "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus",
           "2", "--steps", "2", "--warmup", "3", "--workload", "ffn512_cal", "--cpu-budget", "1"]
    r = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout   # rank 0 alone prints
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["value"] > 0
