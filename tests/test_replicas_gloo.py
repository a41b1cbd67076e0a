"""bench.py's replicas path (one process per GPU, no data-path collective)
on CPU: two gloo ranks agree on the slowest rank's time and on the whole-job
throughput, and under torchrun only rank 0 runs the reference arm."""

import datetime
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        slow = bench.max_over_ranks(10.0 + 5.0 * rank, dist, torch.device("cpu"))
        dist.barrier()
        q.put((rank, slow, bench.job_tok_s(world, 8, 20, slow)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        res = sorted(q.get(timeout=120) for _ in range(world))
    finally:
        for p in procs:
            p.join(timeout=60)
    assert [p.exitcode for p in procs] == [0, 0]
    assert [r[1] for r in res] == [15.0, 15.0]
    # 2 replicas x 8 tokens x 20 steps over the slower rank's 15 ms
    assert all(abs(r[2] - 2 * 8 * 20 / 0.015) < 1e-6 for r in res)


def test_one_gpu_keeps_its_own_time():
    assert bench.max_over_ranks(12.5, None, None) == 12.5
    assert bench.job_tok_s(1, 1, 20, 50.0) == 400.0


def test_reference_arm_runs_on_rank_0_only(monkeypatch):
    called = []
    monkeypatch.setattr(bench, "run_reference", lambda *a, **k: called.append(1))
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2"])
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    assert bench.main() == 0 and called == []
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("LOCAL_RANK", "0")
    assert bench.main() == 0 and called == [1]
