"""Data-parallel Lloyd (points sharded by rows, one all-reduce of float64
sums, counts and objective per iteration) against the single-device fit and
the oracle.  Two ranks run as processes on one GPU and exchange through the
gloo backend (host copies); no kernel of one rank waits on the other."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

N, D, K, ITERS = 24000, 64, 100, 3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem():
    from synth import WORKLOADS, make_problem
    wl = WORKLOADS["1m_k1024"].with_(N=N, D=D, K=K)
    X, C0, _ = make_problem(wl, seed=21, device="cuda")
    return X.contiguous(), C0.contiguous()


def _rank(rank, world, port, q):
    import torch.distributed as dist
    import means_clustering_flashassign_b200 as km
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        X, C0 = _problem()
        rows = slice(rank * N // world, (rank + 1) * N // world)
        r1 = km.fit_data_parallel(X[rows].contiguous(), C0, 1)
        r = km.fit_data_parallel(X[rows].contiguous(), C0, ITERS)
        # numpy arrays travel by value (a torch CPU tensor would be shared by
        # file descriptor, which the parent can only pick up while this
        # process is still alive)
        q.put((rank, r["C"].cpu().numpy(), r["counts"].cpu().numpy(), np.asarray(r["objective"]),
               r["idx"].cpu().numpy(), r1["C"].cpu().numpy()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_match_the_single_device_fit():
    import means_clustering_flashassign_b200 as km
    import oracle
    from tests.parity import CTOL, JTOL, centroid_rel_err

    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted((q.get(timeout=300) for _ in range(world)), key=lambda o: o[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    (_, C_a, n_a, J_a, i_a, C1_a), (_, C_b, n_b, J_b, i_b, _) = out
    # every rank finalises the same sums: identical centroids, counts, objective
    assert np.array_equal(C_a, C_b) and np.array_equal(n_a, n_b) and np.array_equal(J_a, J_b)
    assert int(n_a.sum()) == N
    X, C0 = _problem()
    # the whole point set's objective at t = 1 (same C0 everywhere) equals the oracle's
    _, d1, _ = oracle.assign(X, C0)
    assert abs(J_a[0] - d1.sum()) <= JTOL * d1.sum()
    # after the last iteration: the centroids are the member means of the
    # assignment the ranks made (their rows concatenated)
    idx = np.concatenate([i_a, i_b])
    Cref, cref = oracle.update(X, idx, torch.from_numpy(C_a))
    assert np.array_equal(n_a, cref)
    assert centroid_rel_err(C_a, Cref) <= CTOL["bf16"]
    # the single-device fit agrees: after one iteration (same assignments
    # from C0; float64 sums across ranks here, float32 segments there) the
    # centroids within the accuracy rule, and the last objective within the
    # trajectory bound
    ref1 = km.fit(X, C0, 1)
    ref = km.fit(X, C0, ITERS)
    torch.cuda.synchronize()
    assert centroid_rel_err(C1_a, ref1["C"]) <= CTOL["bf16"]
    assert abs(J_a[-1] - ref["objective"][-1].item()) <= 1e-3 * J_a[-1]
