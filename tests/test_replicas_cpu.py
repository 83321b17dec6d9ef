"""Host side of the multi-GPU path on CPU: two gloo ranks.

Decode shards over independent sequences, so the benchmark runs one replica
per rank with no data-path collective; the only cross-rank steps are the
barriers around the timed region and the max of the per-rank step times.
These tests run those steps as two gloo processes.  The reference arm under
two ranks prints from rank 0 only; rank 1 returns without work.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r"""
import os, sys, types
sys.path.insert(0, os.environ["V4A_ROOT"])
import bench
args = types.SimpleNamespace(impl="ours", gpus=2, steps=1, warmup=3, cpu_seconds=1.0)
world, rank, local = bench.dist_init(args)
assert world == 2 and rank == int(os.environ["RANK"])
bench.barrier(world)
got = bench.max_over_ranks(1.5 + 3.0 * rank, world)
bench.barrier(world)
# the reference arm: only rank 0 may run the oracle; rank 1 must return at once
if rank == 1:
    bench.run_reference(args, world, rank)
print("RESULT", rank, got, flush=True)
import torch.distributed as dist
dist.destroy_process_group()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_take_the_max_step_time():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE="2",
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), V4A_ROOT=ROOT, CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, "-c", WORKER], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.STDOUT, text=True))
    outs = []
    for p in procs:
        try:
            out, _ = p.communicate(timeout=240)
        except subprocess.TimeoutExpired:
            p.kill()
            out, _ = p.communicate()
        outs.append(out)
        assert p.returncode == 0, out
    results = {}
    for out in outs:
        for line in out.splitlines():
            if line.startswith("RESULT"):
                _, r, v = line.split()
                results[int(r)] = float(v)
    assert results == {0: 4.5, 1: 4.5}
    # rank 1 printed no JSON line (the reference arm belongs to rank 0)
    assert not any(line.startswith("{") for line in outs[1].splitlines())


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.25, 1) == 2.25
    bench.barrier(1)  # no-op
