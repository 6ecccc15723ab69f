"""The kernels of one Lloyd iteration chain by programmatic dependent launch
(each becomes resident while the previous one drains and waits on the
device before touching shared data).  The chained fit must give bit-identical
results to plain stream order (KM_PDL=0), through every update path -- the
sorted multi-kernel update with one- and two-pass sorts, and the fused
batched update -- and fit_timed must be fit with a device clock around it."""

import numpy as np
import pytest
import torch

import means_clustering_flashassign_b200 as km
from synth import WORKLOADS, make_problem

pytestmark = pytest.mark.gpu

CASES = [
    dict(N=200_000, D=128, K=1024, B=1),   # one-pass sort, CTA-pair assignment
    dict(N=50_000, D=64, K=5000, B=1),     # two-pass sort (13-bit keys)
    dict(N=70_001, D=32, K=100, B=1),      # ragged tail, small radix
    dict(N=4096, D=64, K=256, B=8),        # fused batched update
]


def _problem(c):
    wl = WORKLOADS["1m_k1024"].with_(**c)
    X, C, _ = make_problem(wl, seed=c["N"] + c["K"], device="cuda")
    return X.contiguous(), C.contiguous()


def _fit(fn, X, C, iters):
    idx = torch.empty(X.shape[:-1], dtype=torch.int32, device=X.device)
    r = fn(X, C, iters, idx_out=idx)
    torch.cuda.synchronize()
    return r, idx


@pytest.mark.parametrize("case", CASES, ids=lambda c: "N{N}_D{D}_K{K}_B{B}".format(**c))
def test_chained_launch_is_bit_identical(case, monkeypatch):
    X, C = _problem(case)
    monkeypatch.setenv("KM_PDL", "0")
    plain, idx_plain = _fit(km.fit, X, C, 4)
    monkeypatch.delenv("KM_PDL")
    chained, idx_chained = _fit(km.fit, X, C, 4)
    assert torch.equal(idx_plain, idx_chained)
    assert torch.equal(plain["C"], chained["C"])
    assert torch.equal(plain["counts"], chained["counts"])
    assert torch.equal(plain["objective"], chained["objective"])


@pytest.mark.parametrize("case", CASES[:1] + CASES[-1:], ids=lambda c: "N{N}_B{B}")
def test_fit_timed_is_fit(case):
    X, C = _problem(case)
    ref, idx_ref = _fit(km.fit, X, C, 3)
    timed, idx_timed = _fit(km.fit_timed, X, C, 3)
    assert timed["iters_ms"] > 0.0
    assert torch.equal(idx_ref, idx_timed)
    assert torch.equal(ref["C"], timed["C"])
    assert torch.equal(ref["objective"], timed["objective"])
    zero = km.fit_timed(X, C, 0)
    assert zero["iters_ms"] == 0.0


@pytest.mark.parametrize("K", [100, 300, 1024, 5000])
@pytest.mark.parametrize("iters", [1, 2, 3])
def test_fit_centroids_are_member_means_of_its_assignment(K, iters):
    """After a fit of any length, C_out is the member mean (float64 here) of
    the assignment the fit returns, and counts its sizes: the update of the
    last iteration saw exactly the assignment kernel's output, whatever the
    launch chaining let overlap."""
    wl = WORKLOADS["1m_k1024"].with_(N=30000, D=128, K=K, B=1, dtype="bf16")
    X, C0, _ = make_problem(wl, seed=5, device="cuda")
    X, C0 = X.contiguous(), C0.contiguous()
    r, idx = _fit(km.fit, X, C0, iters)
    idx = idx.cpu().numpy()
    cnt = np.bincount(idx, minlength=K)
    assert np.array_equal(r["counts"].cpu().numpy(), cnt)
    sums = np.zeros((K, 128))
    np.add.at(sums, idx, X.float().cpu().numpy())
    ok = cnt > 0
    C = r["C"].cpu().numpy().astype(np.float64)
    err = np.abs(sums[ok] / cnt[ok, None] - C[ok]).max()
    assert err <= 1e-4, err
