"""The benchmark's multi-process path on CPU (gloo, world size 2): the
reference arm prints one line from rank 0 only, and the timing reduction
takes the maximum over ranks."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_reference_arm_two_ranks():
    port = _free_port()
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    cmd = ["timeout", "-k", "30", "240", sys.executable, "-m", "torch.distributed.run",
           "--nnodes=1", "--nproc-per-node=2", "--master-addr=127.0.0.1",
           f"--master-port={port}", os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--workload", "tiny", "--gpus", "2", "--steps", "2", "--warmup", "1",
           "--cpu-seconds", "1"]
    res = subprocess.run(cmd, capture_output=True, text=True, cwd=ROOT, env=env)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["value"] > 0 and rec["steps"] == 2
    assert rec["unit"] == "TFLOP/s" and rec["higher_is_better"] is True
    assert rec["n_gpus"] == 2 and rec["warmup"] == 1 and rec["config"]["workload"] == "tiny"
    assert rec["cpu_baseline"]["kind"] == "oracle"
    assert rec["e2e"]["h2d_bytes_per_step"] == 0
    # the same config object as the GPU arm's line
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W
    wl = W.WORKLOADS["tiny"]
    assert rec["config"] == bench.bench_config(wl, 0.99, max(1, wl.sparse_steps), 2)


def _worker(rank, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE="2", LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=2)
    try:
        bench.barrier(2)
        out[rank] = bench.max_over_ranks(1.5 + rank, 2)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_worker, args=(port, out), nprocs=2, start_method="spawn", join=True)
    assert dict(out) == {0: 2.5, 1: 2.5}


def test_list_schedule_makespan():
    """The in-order list scheduling the scheduler analysis simulates: each
    job goes, in order, to the worker that becomes free first."""
    sys.path.insert(0, ROOT)
    import bench
    assert bench._list_schedule([3, 3, 3, 3], 2) == 6
    assert bench._list_schedule([5, 1, 1, 1, 1, 1], 2) == 5
    assert bench._list_schedule([1, 1, 1, 1, 1, 5], 2) == 7   # a long job last sets the tail
    assert bench._list_schedule([2.5], 4) == 2.5
