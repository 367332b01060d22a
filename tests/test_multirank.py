"""Multi-process (world size 2) checks of the benchmark's host-side rank logic
on CPU, over the gloo backend: the job's time is the slowest rank's, its
throughput counts every rank's work (weak scaling), and under a 2-rank launch
only rank 0 prints the reference arm's line."""
import json
import multiprocessing as mp
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


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r took (r + 1) * 10 ms for the steps and 5 - r ms for the forward
        tot, fwd = bench.max_over_ranks([(rank + 1) * 10.0, 5.0 - rank])
        q.put((rank, tot, fwd, bench.job_tflops(world, 1e12, 4, tot)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, tot, fwd, tflops in out:
        assert tot == 20.0 and fwd == 5.0          # max over ranks, on every rank
        # 2 ranks x 4 steps x 1 TFLOP in 20 ms
        assert abs(tflops - 2 * 4 * 1e12 / 20e-3 / 1e12) < 1e-9


def test_single_process_timings_pass_through():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.5]) == [3.0, 4.5]
    assert abs(bench.job_tflops(1, 2e12, 3, 6.0) - 1000.0) < 1e-9


def test_reference_arm_prints_once_under_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--workload", "1", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    assert lines[0]["impl"] == "reference" and lines[0]["n_gpus"] == 2
    assert lines[0]["value"] > 0
