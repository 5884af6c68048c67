"""The N > 1 path of bench.py on CPU with two gloo ranks: the job's time is the
slowest rank's, the metric counts the chunks of every rank (replicas, weak
scaling), and the reference arm runs on rank 0 only."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 * (rank + 1)          # rank 1 is the slowest
        ms = bench.max_over_ranks(local_ms, world, "cpu")
        q.put((rank, ms, bench.ms_per_chunk(ms, steps=4, batch_per_rank=1, world=world)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_count_all_chunks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ps = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ms, per_chunk in got:
        assert ms == 20.0                      # every rank agrees on the slowest time
        assert per_chunk == 20.0 / (4 * 1 * 2)  # chunks of both replicas count


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.ms_per_chunk(8.0, steps=2, batch_per_rank=4, world=1) == 1.0


def test_reference_arm_prints_on_rank_zero_only(capsys):
    class A:
        steps, warmup, gpus = 1, 0, 2
    bench.reference_arm(A(), rank=1)
    assert capsys.readouterr().out == ""
