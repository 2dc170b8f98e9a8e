"""Multi-rank plumbing of bench.py on CPU: two gloo ranks.

bench.py runs one process per GPU; heads and batches are independent, so every
rank runs its own copy of the workload and the only exchange is the timing:
a barrier around the timed region and the slowest rank's time (max over
ranks). These tests run that plumbing with the gloo backend on CPU, and the
reference arm's rule that under several ranks only rank 0 runs and prints.
"""
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


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, ms_local, queue):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        cpu = torch.device("cpu")
        bench.barrier(world)
        slowest = bench.max_over_ranks(ms_local[rank], world, cpu)
        rate, ms_step = bench.weak_scaling_rate(1000, ms_local[rank], world, cpu, steps=4)
        bench.barrier(world)
        queue.put((rank, slowest, rate, ms_step))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_rank():
    world, port = 2, free_port()
    ms_local = [8.0, 10.0]           # rank 1 is slower
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, ms_local, queue))
             for r in range(world)]
    for p in procs:
        p.start()
    results = [queue.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, rate, ms_step in results:
        assert slowest == 10.0
        assert ms_step == pytest.approx(2.5)                   # 10 ms over 4 steps
        assert rate == pytest.approx(1000 * 2 / 2.5e-3)        # both ranks' units / slowest time


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    rate, ms = bench.weak_scaling_rate(64, 2.0, 1, torch.device("cpu"), steps=2)
    assert ms == 1.0 and rate == pytest.approx(64e3)


def test_reference_arm_prints_on_rank0_only():
    """Launched as torchrun would (RANK / WORLD_SIZE in the environment): rank 0 times
    the oracle and prints one JSON line, rank 1 exits 0 without work."""
    outs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1")
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                            "--gpus", "2", "--steps", "1", "--warmup", "0",
                            "--cpu-tokens-ref", "64"],
                           cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
        assert r.returncode == 0, r.stderr
        outs.append(r.stdout.strip())
    assert outs[1] == ""
    line = json.loads(outs[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
