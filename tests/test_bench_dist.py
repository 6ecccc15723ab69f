"""The bench's multi-rank host logic on CPU: two gloo ranks, as torchrun would
launch them (RANK / WORLD_SIZE / MASTER_* in the environment).  Each rank runs
its own replica problem with no data-path collective; the job's time is the
slowest rank's, and only rank 0 reports (the reference arm on rank 0 alone)."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        ms = [12.5, 20.0][rank]  # rank 1 is the slow one
        ms_max = bench.max_over_ranks(world, ms, device="cpu")
        args = type("A", (), {"workload": "small_f32", "cpu_sample": 256, "steps": 1, "warmup": 3, "seed": 0})()
        ref = bench.run_reference(args, world, rank) if rank == 1 else "skipped"
        q.put((rank, ms_max, bench.job_rate(10, world, ms_max), ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_and_rank0_reports():
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
    assert [o[1] for o in out] == [20.0, 20.0]           # both ranks see the max
    assert out[0][2] == pytest.approx(10 * 2 / 0.020)    # 2 x 10 iterations in 20 ms
    assert out[1][3] is None                             # the reference arm runs on rank 0 only


def test_single_rank_passes_time_through():
    assert bench.max_over_ranks(1, 3.5) == 3.5
    assert bench.job_rate(20, 1, 10.0) == pytest.approx(2000.0)
