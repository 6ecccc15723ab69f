"""The out-of-core workloads at their stated sizes ("Flash-KMeans", §2.3
Chunked Stream Overlap: the streamed fit must give the in-core result; §4
Results runs one billion points, beyond the device's memory).

ooc_268m_k4096: N = 268,435,456 bf16 points of D = 128 (64 GiB) in pinned
host memory, K = 4096, streamed in 16M-row chunks with copy/compute overlap.
ooc_1b_k4096: N = 2^30 points (256 GiB, never held whole), streamed through
km_fit_source from a 2^28-row pinned pool (row i = pool row i mod 2^28).

The oracle cannot evaluate all N x K distances, so the first Lloyd iteration
is checked on what it can compute one by one and on properties that hold at
any size:
  * a seeded sample of 4096 rows: the device's assignment under C0 against
    the oracle's argmin (the parity gap rule);
  * the counts are the histogram of the assignment and sum to N;
  * 16 sampled clusters and the largest: the device's centroid is the
    float64 mean of all its members, gathered chunk by chunk on the host;
  * the objective J_1 against the oracle's direct-form sum of squared
    distances of every point to its assigned centroid (float64, all points);
  * one billion points: every copy of a pool row gets the same cluster, and
    counts and objective are four times the pool's.
Needs ~72 GiB of available host memory; the one-billion-point case runs only
with KM_FULL_SIZE=1 (it streams 256 GiB per iteration)."""

import os

import numpy as np
import pytest
import torch

import means_clustering_flashassign_b200 as km
import oracle
from synth import WORKLOADS, init_rows, make_points, pool_workload
from tests.parity import CTOL, JTOL, centroid_rel_err, check_assignment

pytestmark = pytest.mark.gpu
CHUNK = 16 << 20


def _mem_available_gib():
    with open("/proc/meminfo") as f:
        for line in f:
            if line.startswith("MemAvailable:"):
                return int(line.split()[1]) / 2**20
    return 0.0


def _pool(wl):
    pw = pool_workload(wl)
    need = pw.N * pw.D * 2 / 2**30 + 8
    have = _mem_available_gib()
    if have < need:
        pytest.skip(f"needs about {need:.0f} GiB of available host memory, the host has {have:.0f} GiB")
    dev = torch.device("cuda", 0)
    Xh = torch.empty((pw.N, pw.D), dtype=torch.bfloat16, pin_memory=True)
    make_points(pw, seed=0, device=dev, out=Xh)
    sel = init_rows(wl, 0, dev).cpu()
    return Xh, Xh[sel].to(dev).contiguous()


def _check_first_iteration(wl, Xh, C0, idx, counts, C1, J1, copies=1):
    """idx: the assignment of the pool's rows (numpy), counts/C1/J1 those of
    the fit over `copies` copies of the pool."""
    P = Xh.shape[0]
    C0h = C0.cpu()
    # sampled rows: the assignment under C0 against the oracle
    rows = np.sort(np.random.default_rng(5).choice(P, size=4096, replace=False))
    check_assignment(Xh[torch.from_numpy(rows)], C0h, idx[rows], None, "bf16")
    # counts: the histogram of the assignment
    assert int(counts.sum()) == copies * P
    assert np.array_equal(counts, copies * np.bincount(idx, minlength=wl.K))
    # member means of sampled clusters and the largest, over all points
    hot = int(np.argmax(counts))
    clusters = np.array(sorted(set(np.random.default_rng(6).choice(wl.K, 16, replace=False).tolist()) | {hot}))
    relabel = np.full(wl.K, -1, np.int64)
    relabel[clusters] = np.arange(clusters.size)
    members, labels = [], []
    for c0 in range(0, P, CHUNK):
        ic = idx[c0:c0 + CHUNK]
        m = np.nonzero(relabel[ic] >= 0)[0]
        members.append(Xh[c0:c0 + CHUNK][torch.from_numpy(m)])
        labels.append(relabel[ic[m]].astype(np.int32))
    Cref, cnt = oracle.update(torch.cat(members), np.concatenate(labels), C1[torch.from_numpy(clusters)])
    assert np.array_equal(copies * cnt, counts[clusters])
    assert centroid_rel_err(C1[torch.from_numpy(clusters)], Cref) <= CTOL["bf16"]
    # J_1: every point's direct-form distance to its assigned centroid
    Jref = 0.0
    for c0 in range(0, P, CHUNK):
        Jref += oracle.objective_assigned_bf16(Xh[c0:c0 + CHUNK], C0h, idx[c0:c0 + CHUNK])
    Jref *= copies
    assert abs(J1 - Jref) <= JTOL * Jref, (J1, Jref)


def test_out_of_core_full_size_first_iteration():
    wl = WORKLOADS["ooc_268m_k4096"]
    Xh, C0 = _pool(wl)
    r = km.fit_host(Xh, C0, 1, CHUNK, want_idx=True)
    torch.cuda.synchronize()
    _check_first_iteration(wl, Xh, C0, r["idx"].cpu().numpy(), r["counts"].cpu().numpy(), r["C"].cpu(),
                           float(r["objective"][0]))


@pytest.mark.skipif(os.environ.get("KM_FULL_SIZE") != "1", reason="one billion points: set KM_FULL_SIZE=1")
def test_one_billion_points_first_iteration():
    wl = WORKLOADS["ooc_1b_k4096"]
    Xh, C0 = _pool(wl)
    P = Xh.shape[0]
    copies = wl.N // P

    def source(row0, rows, slot):
        r = row0 % P
        return Xh[r:r + rows]

    r = km.fit_source(source, wl.N, C0, 1, CHUNK, want_idx=True)
    torch.cuda.synchronize()
    idx = r["idx"]
    for j in range(1, copies):  # every copy of a pool row gets the same cluster
        assert torch.equal(idx[j * P:(j + 1) * P], idx[:P])
    _check_first_iteration(wl, Xh, C0, idx[:P].cpu().numpy(), r["counts"].cpu().numpy(), r["C"].cpu(),
                           float(r["objective"][0]), copies=copies)
