"""The bench's multi-rank host logic on CPU: two gloo ranks, as torchrun would
launch them (RANK / WORLD_SIZE / MASTER_* in the environment).  The job's time
is the slowest rank's, only rank 0 reports (the reference arm on rank 0
alone), the data-parallel shards tile the whole point set, and both arms
describe the workload with the same config object."""

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
        args = type("A", (), {"workload": "small_f32", "ref_seconds": 0.5, "steps": 1, "warmup": 3, "seed": 0})()
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


def test_shards_tile_the_whole_problem():
    for world in (1, 2, 3, 8):
        rows = [bench.shard_rows(1000, world, r) for r in range(world)]
        assert rows[0].start == 0 and rows[-1].stop == 1000 * world
        assert all(a.stop == b.start for a, b in zip(rows, rows[1:]))


def test_repeats_reach_the_minimum_timed_region():
    assert bench.repeats_for(1.0, 160.0) == 8          # 8 x 160 ms >= 1.15 s (margin for the clock)
    assert bench.repeats_for(1.0, 2000.0) == 1
    assert bench.repeats_for(1.0, 6.2) * 6.2 >= 1150.0
    # a warm-up estimate 10 % faster than the capped rate still reaches 1 s
    assert bench.repeats_for(1.0, 166.5 / 1.1) * 166.5 >= 1000.0


def test_both_arms_share_the_config_object():
    from synth import WORKLOADS
    wl = WORKLOADS["4m_k16384_zipf"]
    a = bench.workload_config(wl, 1, "single")
    assert a == bench.workload_config(wl, 1, "single")
    assert a["workload"] == "4m_k16384_zipf" and a["K"] == 16384 and "zipf1.2" in a["mixture"]
    assert "larger than L2" in a["l2"]
    small = bench.workload_config(WORKLOADS["small_f32"], 1, "single")
    assert "fits in L2" in small["l2"]


def test_reference_arm_reports_the_same_config_as_ours():
    args = type("A", (), {"workload": "small_f32", "ref_seconds": 0.5, "steps": 2, "warmup": 3, "seed": 0})()
    ref = bench.run_reference(args, 1, 0)
    from synth import WORKLOADS
    assert ref["config"] == bench.workload_config(WORKLOADS["small_f32"], 1, "single")
    assert ref["impl"] == "reference" and ref["unit"] == bench.UNIT and ref["e2e"]["value"] == ref["value"]
    assert ref["cpu_baseline"]["kind"] == "oracle" and ref["cpu_baseline"]["cores"] >= 1


def test_traffic_record_roundtrip(tmp_path, monkeypatch):
    csv = tmp_path / "raw.csv"
    csv.write_text('"ID","Kernel Name","dram__bytes_read.sum","dram__bytes_write.sum"\n'
                   '"","","Mbyte","Mbyte"\n'
                   '"0","void km::k_assign<256, 0, 1, 0>(...)","300.5","7.5"\n'
                   '"1","void km::k_assign<256, 0, 1, 0>(...)","301.5","7.5"\n'
                   '"2","void km::k_segsum<16, 1>(...)","280","1"\n')
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "traffic.json"))
    e = bench.record_traffic(str(csv), "k_assign", "1m_k1024", 2.0, "ncu ...")
    assert e["bytes_per_launch"] == round((308e6 + 309e6) / 2 * 2.0) and e["launches_captured"] == 2
    assert bench.recorded_traffic("k_assign", "1m_k1024") == e["bytes_per_launch"]
    assert bench.recorded_traffic("k_assign", "4m_k16384_zipf") is None
    monkeypatch.setattr(bench, "kernel_source_sha", lambda k="k_assign": "0000000000000000")
    assert bench.recorded_traffic("k_assign", "1m_k1024") is None  # sources changed since the capture
