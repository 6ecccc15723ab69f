"""Full-size parity on the benchmark workloads, in the launch configuration the
bench times (the fit entry points), checked on sampled outputs the oracle can
compute one by one and on properties that hold at any size."""

import numpy as np
import pytest
import torch

import means_clustering_flashassign_b200 as km
import oracle
from synth import WORKLOADS, make_problem
from tests.parity import CTOL, JTOL, centroid_rel_err, check_assignment, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _sample_rows(n, m, seed):
    return np.sort(np.random.default_rng(seed).choice(n, size=min(m, n), replace=False))


def _check_clusters_are_member_means(X, idx, C, clusters, kind):
    idx_np = idx.cpu().numpy()
    Cn = C.cpu()
    for k in clusters:
        mem = np.nonzero(idx_np == k)[0]
        if mem.size == 0:
            continue
        Xk = X[torch.from_numpy(mem).to(X.device)]
        Cref, cnt = oracle.update(Xk, np.zeros(mem.size, np.int32), Cn[k:k + 1])
        assert cnt[0] == mem.size
        assert centroid_rel_err(Cn[k:k + 1], Cref) <= CTOL[kind], k


@pytest.mark.parametrize("name,rows_sample", [("1m_k1024", 4096), ("4m_k16384_zipf", 1536)])
def test_single_problem_workload(name, rows_sample):
    wl = WORKLOADS[name]
    X, C0, _ = make_problem(wl, seed=0, device=DEV)
    X, C0 = X.contiguous(), C0.contiguous()
    # step 1 through the separate entry points, sampled against the oracle
    idx, md, obj = km.assign(X, C0)
    torch.cuda.synchronize()
    rows = _sample_rows(wl.N, rows_sample, 1)
    check_assignment(X[torch.from_numpy(rows).to(DEV)], C0, idx[torch.from_numpy(rows).to(DEV)],
                     md[torch.from_numpy(rows).to(DEV)], "bf16")
    assert abs(obj.item() - md.double().sum().item()) <= 1e-9 * obj.item()
    C1, counts = km.update(X, idx, C0.float().clone())
    torch.cuda.synchronize()
    assert int(counts.sum()) == wl.N
    assert torch.equal(counts.cpu(), torch.bincount(idx.long().cpu(), minlength=wl.K).int())
    rng = np.random.default_rng(2)
    hot = int(torch.argmax(counts).item())
    clusters = sorted(set(rng.choice(wl.K, 24, replace=False).tolist()) | {hot})
    _check_clusters_are_member_means(X, idx, C1, clusters, "bf16")
    # the bench's launch configuration: the fit loop with per-phase events
    r = km.fit_profile(X, C0, 3)
    assert abs(r["objective"][0].item() - obj.item()) <= 1e-12 * obj.item()  # same tiles, another sum order
    J = r["objective"].cpu().numpy()
    assert np.all(np.diff(J) < 0)
    Cf = r["C"]
    # second fit with idx kept: the final centroids are the member means
    r2 = km.fit(X, C0, 3)
    torch.cuda.synchronize()
    assert torch.equal(r2["C"], Cf)
    _check_clusters_are_member_means(X, r2["idx"], r2["C"], clusters, "bf16")


def test_batched_workload_full_size():
    wl = WORKLOADS["batch512_k256"]
    X, C0, _ = make_problem(wl, seed=0, device=DEV)
    r = km.fit(X.contiguous(), C0.contiguous(), wl.iters)
    torch.cuda.synchronize()
    rp = km.fit(X.contiguous(), C0.contiguous(), wl.iters - 1)
    torch.cuda.synchronize()
    for b in [0, 1, 77, 255, 300, 511]:
        ref = oracle.fit(X[b], C0[b], wl.iters, mirror="bf16")
        J = r["objective"][b].cpu().numpy()
        assert abs(J[0] - ref["J"][0]) <= JTOL * ref["J"][0]
        _, d1, _ = oracle.assign(X[b], rp["C"][b].to(torch.bfloat16))
        assert abs(J[-1] - d1.sum()) <= JTOL * d1.sum()
        assert abs(J[-1] - ref["J"][-1]) <= 1e-3 * ref["J"][-1]
        Cchk, cchk = oracle.update(X[b], r["idx"][b].cpu().numpy(), r["C"][b])
        assert np.array_equal(r["counts"][b].cpu().numpy(), cchk)
        assert centroid_rel_err(r["C"][b], Cchk) <= CTOL["bf16"]


def test_small_f32_workload_full_trajectory():
    wl = WORKLOADS["small_f32"]
    X, C0, _ = make_problem(wl, seed=0, device=DEV)
    r = km.fit(X, C0, wl.iters)
    torch.cuda.synchronize()
    ref = oracle.fit(X, C0, wl.iters, mirror="f32")
    J = r["objective"].cpu().numpy()
    assert abs(J[0] - ref["J"][0]) <= JTOL * ref["J"][0]
    assert abs(J[-1] - ref["J"][-1]) <= 1e-3 * ref["J"][-1]
    Cchk, _ = oracle.update(X, r["idx"].cpu().numpy(), r["C"])
    assert centroid_rel_err(r["C"], Cchk) <= CTOL["f32"]


def test_host_resident_stream_scaled():
    """The out-of-core workload's chunking (16M-row chunks) on a 40M-point
    instance that also fits on the device: the streamed fit equals the
    in-core fit."""
    wl = WORKLOADS["ooc_268m_k4096"].with_(N=40_000_000, host_resident=False)
    X, C0, _ = make_problem(wl, seed=0, device=DEV)
    ref = km.fit(X, C0, 2)
    torch.cuda.synchronize()
    Xh = torch.empty(X.shape, dtype=X.dtype, pin_memory=True)
    Xh.copy_(X)
    out = km.fit_host(Xh, C0, 2, chunk_rows=16 << 20, want_idx=True)
    np.testing.assert_allclose(out["objective"].numpy()[:1], ref["objective"].cpu().numpy()[:1], rtol=JTOL)
    np.testing.assert_allclose(out["objective"].numpy(), ref["objective"].cpu().numpy(), rtol=1e-3)
    # streamed centroids are the member means of the streamed final assignment
    hot = int(torch.argmax(out["counts"]).item())
    clusters = sorted(set(np.random.default_rng(3).choice(wl.K, 8, replace=False).tolist()) | {hot})
    _check_clusters_are_member_means(X, out["idx"], out["C"], clusters, "bf16")
    assert int(out["counts"].sum()) == wl.N
