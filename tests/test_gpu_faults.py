"""Host-side fault injection (KM_FAULT) on the GPU: each injection point makes
its call fail cleanly with KM_ERR_INJECTED before the failing step is issued.
Nothing faults, traps or hangs the GPU: the injector only skips a host call.
Afterwards the same workspace and context give results bit-identical to a
fit made before the failure (the context is usable, the workspace state
left by the aborted call does not leak into the next call), and repeated
failures of the out-of-core fit do not exhaust streams or events."""

import numpy as np
import pytest
import torch

import means_clustering_flashassign_b200 as km
from synth import WORKLOADS, make_problem

pytestmark = pytest.mark.gpu

INJECTED = 6


def _problem(N=40_000, D=128, K=300, seed=2):
    wl = WORKLOADS["1m_k1024"].with_(N=N, D=D, K=K)
    X, C0, _ = make_problem(wl, seed=seed, device="cuda")
    return X.contiguous(), C0.contiguous()


def _same(a, b):
    for k in ("C", "counts", "objective"):
        assert torch.equal(torch.as_tensor(a[k]).cpu(), torch.as_tensor(b[k]).cpu()), k


def _expect_injected(fn):
    with pytest.raises(km.KMError) as e:
        fn()
    assert e.value.status == INJECTED, e.value
    assert "injected" in e.value.message


@pytest.mark.parametrize("spec", ["launch", "launch:4", "launch:13"])
def test_fit_launch_fault(spec, monkeypatch):
    X, C0 = _problem()
    ws = torch.empty(km.workspace_size(km.OP_FIT, 1, X.shape[0], 128, 300, km.BF16), dtype=torch.uint8,
                     device="cuda")
    ref = km.fit(X, C0, 3, workspace=ws)
    torch.cuda.synchronize()
    ref = {k: v.clone() for k, v in ref.items() if v is not None}
    monkeypatch.setenv("KM_FAULT", spec)
    _expect_injected(lambda: km.fit(X, C0, 3, workspace=ws))
    monkeypatch.delenv("KM_FAULT")
    again = km.fit(X, C0, 3, workspace=ws)
    torch.cuda.synchronize()
    _same(again, ref)


@pytest.mark.parametrize("spec", ["alloc", "alloc:3", "h2d", "h2d:3", "launch:2", "launch:9"])
def test_fit_host_faults(spec, monkeypatch):
    X, C0 = _problem()
    Xh = X.cpu().pin_memory()
    ref = km.fit_host(Xh, C0, 2, chunk_rows=9000)
    monkeypatch.setenv("KM_FAULT", spec)
    _expect_injected(lambda: km.fit_host(Xh, C0, 2, chunk_rows=9000))
    monkeypatch.delenv("KM_FAULT")
    _same(km.fit_host(Xh, C0, 2, chunk_rows=9000), ref)


def test_repeated_fit_host_failures_release_their_streams_and_events(monkeypatch):
    X, C0 = _problem(N=12_000, K=50)
    Xh = X.cpu().pin_memory()
    ref = km.fit_host(Xh, C0, 1, chunk_rows=4000)
    monkeypatch.setenv("KM_FAULT", "h2d:2")
    for _ in range(300):
        _expect_injected(lambda: km.fit_host(Xh, C0, 1, chunk_rows=4000))
    monkeypatch.delenv("KM_FAULT")
    _same(km.fit_host(Xh, C0, 1, chunk_rows=4000), ref)


@pytest.mark.parametrize("call,spec", [("profile", "alloc:2"), ("timed", "alloc"), ("timed", "launch:3"),
                                       ("assign", "launch:2"), ("update", "launch:2")])
def test_other_entry_points(call, spec, monkeypatch):
    X, C0 = _problem()
    fns = {
        "profile": lambda: km.fit_profile(X, C0, 2),
        "timed": lambda: km.fit_timed(X, C0, 2),
        "assign": lambda: km.assign(X, C0),
        "update": lambda: km.update(X, torch.zeros(X.shape[0], dtype=torch.int32, device="cuda"),
                                    C0.float().clone()),
    }
    monkeypatch.setenv("KM_FAULT", spec)
    _expect_injected(fns[call])
    monkeypatch.delenv("KM_FAULT")
    out = fns[call]()
    torch.cuda.synchronize()
    assert out is not None


def test_unknown_fault_point_is_ignored(monkeypatch):
    X, C0 = _problem(N=5000, K=20)
    monkeypatch.setenv("KM_FAULT", "disk:1")
    r = km.fit(X, C0, 2)
    torch.cuda.synchronize()
    assert np.isfinite(r["objective"].cpu().numpy()).all()
