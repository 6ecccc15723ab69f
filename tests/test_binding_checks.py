"""Host-side checks of the Python binding, no GPU needed.

Every tensor the kernels read or write must be on the points' device, of the
dtype and shape the call writes, and contiguous; a caller-supplied stream must
be on the same device.  A short idx or mindist would let a kernel write past
its end, and a tensor on another GPU would be read through a tensor map that
covers the wrong device's memory, so these are rejected before any call into
the library.  The data-parallel exchange packs sums, counts and the objective
into one float64 buffer added by a single all-reduce; two gloo ranks check it
on the CPU."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import means_clustering_flashassign_b200 as km

CPU = torch.device("cpu")


def test_tensor_check_accepts_a_matching_tensor():
    t = torch.empty(7, dtype=torch.int32)
    assert km._check_tensor(t, "idx", CPU, torch.int32, (7,)) is t


@pytest.mark.parametrize("bad,msg", [
    (torch.empty(7, dtype=torch.int64), "must be torch.int32"),          # wrong dtype
    (torch.empty(6, dtype=torch.int32), "must have shape"),              # too short: the kernel would overrun it
    (torch.empty(14, dtype=torch.int32)[::2], "contiguous"),             # strided view
    (torch.empty(7, dtype=torch.int32, device="meta"), "the points are on"),  # another device
])
def test_tensor_check_rejects(bad, msg):
    with pytest.raises(ValueError, match=msg):
        km._check_tensor(bad, "idx", CPU, torch.int32, (7,))


def test_stream_on_another_device_is_rejected():
    class FakeStream:
        device = torch.device("cuda", 1)
    with pytest.raises(ValueError, match="stream"):
        km._check_stream(FakeStream(), torch.device("cuda", 0))
    km._check_stream(None, torch.device("cuda", 0))


@pytest.mark.parametrize("call", [
    lambda X, C: km.assign(X, C),
    lambda X, C: km.assign_static(X, C),
    lambda X, C: km.fit(X, C, 2),
    lambda X, C: km.fit_timed(X, C, 2),
    lambda X, C: km.fit_profile(X, C, 2),
    lambda X, C: km.update(X, torch.zeros(X.shape[0], dtype=torch.int32), C.float()),
    lambda X, C: km.ablation_assign_materialized(X, C),
])
def test_host_tensors_are_rejected_before_the_library(call):
    X = torch.randn(64, 16).to(torch.bfloat16)
    C = X[:4].clone()
    with pytest.raises(ValueError, match="CUDA"):
        call(X, C)


def test_pack_layout_is_one_contiguous_float64_buffer():
    lay = km.pack_layout(5, 3)
    assert lay["size"] == 5 * 3 + 5 + 1
    assert (lay["sums"].start, lay["sums"].stop) == (0, 15)
    assert (lay["counts"].start, lay["counts"].stop) == (15, 20)
    assert (lay["objective"].start, lay["objective"].stop) == (20, 21)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        K, D = 4, 3
        lay = km.pack_layout(K, D)
        buf = torch.zeros(lay["size"], dtype=torch.float64)
        # rank r's shard: sums (r + 1) * [0 .. KD), counts r + k, objective 10^r
        buf[lay["sums"]] = (rank + 1) * torch.arange(K * D, dtype=torch.float64)
        buf[lay["counts"]] = rank + torch.arange(K, dtype=torch.float64)
        buf[lay["objective"]] = 10.0 ** rank
        km.exchange_packed(buf)
        q.put((rank, buf.tolist()))
    finally:
        dist.destroy_process_group()


def test_packed_exchange_adds_sums_counts_and_objective_in_one_all_reduce():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    K, D = 4, 3
    want = [3.0 * i for i in range(K * D)] + [1.0 + 2 * k for k in range(K)] + [11.0]
    assert out[0] == want and out[1] == want


def test_exchange_rejects_a_buffer_of_another_dtype():
    with pytest.raises(ValueError, match="float64"):
        km.exchange_packed(torch.zeros(4, dtype=torch.float32))
