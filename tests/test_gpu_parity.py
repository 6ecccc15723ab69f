"""GPU parity: every step of the CUDA path (through the C ABI) against the
CPU oracle on the same seeded inputs, at sizes the oracle finishes in seconds
that span several tiles and ragged tails, plus the method's edge cases."""

import numpy as np
import pytest
import torch

import means_clustering_flashassign_b200 as km
import oracle
from synth import WORKLOADS, make_problem
from tests.parity import CTOL, JTOL, centroid_rel_err, check_assignment, f64

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _mixture(N, D, K, dtype, seed=0, B=1, sigma=1.0, weights="equal"):
    wl = WORKLOADS["1m_k1024"].with_(N=N, D=D, K=K, B=B, dtype=dtype, sigma=sigma, weights=weights,
                                     centers="normal2" if dtype == "bf16" else "uniform10")
    X, C0, _ = make_problem(wl, seed=seed, device=DEV)
    return X.contiguous(), C0.contiguous()


ASSIGN_BF16 = [(1000, 64, 10), (5000, 128, 1024), (3001, 128, 300), (20000, 128, 1000), (2000, 256, 100),
               (777, 8, 7), (4096, 96, 257), (129, 16, 1), (130, 32, 130), (500, 64, 64), (70000, 128, 513)]


@pytest.mark.parametrize("N,D,K", ASSIGN_BF16)
def test_assign_bf16(N, D, K):
    X, C = _mixture(N, D, K, "bf16", seed=N + K)
    idx, md, obj = km.assign(X, C)
    torch.cuda.synchronize()
    r = check_assignment(X, C, idx, md, "bf16")
    assert r["n_clear"] > 0.5 * r["n"]
    J = r["d1"].sum()
    assert abs(obj.item() - J) <= JTOL * J + r["jfloor"]


ASSIGN_F32 = [(16384, 32, 64), (3000, 64, 100), (1000, 8, 5), (1000, 40, 70), (257, 32, 257), (5000, 16, 300)]


@pytest.mark.parametrize("N,D,K", ASSIGN_F32)
def test_assign_f32_tf32_split(N, D, K):
    X, C = _mixture(N, D, K, "f32", seed=N + D)
    idx, md, obj = km.assign(X, C)
    torch.cuda.synchronize()
    r = check_assignment(X, C, idx, md, "f32")
    assert r["n_clear"] > 0.9 * r["n"]
    J = r["d1"].sum()
    assert abs(obj.item() - J) <= JTOL * J + r["jfloor"]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_assign_integer_data_exact_with_ties(dtype):
    """Integer coordinates make every product and score exact in both paths,
    so the argmin (lowest index on exact ties) and the distance must match
    the oracle bit for bit; duplicated centroids must never win over the
    first copy."""
    g = torch.Generator().manual_seed(7)
    N, D, K = 3000, 64 if dtype == "bf16" else 32, 200
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    X = torch.randint(-3, 4, (N, D), generator=g).to(tdt)
    C = torch.randint(-3, 4, (K, D), generator=g).to(tdt)
    C[100:150] = C[0:50]          # exact duplicates at higher indices
    C[199] = C[3]
    X[:50] = C[:50]               # points sitting exactly on centroids
    Xg, Cg = X.to(DEV), C.to(DEV)
    idx, md, _ = km.assign(Xg, Cg)
    io, d1, _ = oracle.assign(X, C)
    assert np.array_equal(idx.cpu().numpy(), io)
    assert np.array_equal(md.cpu().double().numpy(), d1)
    assert not np.isin(idx.cpu().numpy(), np.r_[100:150, 199]).any()


def test_assign_batched_instances():
    X, C = _mixture(1000, 64, 40, "bf16", B=3, seed=3)
    idx, md, obj = km.assign(X, C)
    torch.cuda.synchronize()
    for b in range(3):
        r = check_assignment(X[b], C[b], idx[b], md[b], "bf16")
        assert abs(obj[b].item() - r["d1"].sum()) <= JTOL * r["d1"].sum() + r["jfloor"]


@pytest.mark.parametrize("N,K,kind", [(100000, 1024, "uniform"), (50000, 16384, "zipf"), (7777, 5000, "uniform"),
                                      (4096, 1, "uniform"), (12345, 300, "empty"), (3, 2, "uniform"),
                                      (300000, 4096, "hot"), (65536, 300, "hot"), (65537, 300, "hot"),
                                      (65536, 8192, "zipf"), (700001, 1024, "zipf"), (700001, 9000, "hot")])
def test_argsort_is_the_stable_inverse_map(N, K, kind):
    rng = np.random.default_rng(N + K)
    if kind == "zipf":
        w = np.arange(1, K + 1) ** -1.2
        idx = rng.choice(K, N, p=w / w.sum())
    elif kind == "empty":
        idx = rng.choice(np.arange(0, K, 3), N)
    elif kind == "hot":
        idx = np.where(rng.random(N) < 0.3, 17, rng.integers(0, K, N))
    else:
        idx = rng.integers(0, K, N)
    idx = idx.astype(np.int32)
    perm, start = km.argsort(torch.from_numpy(idx).to(DEV), K)
    ref_perm, ref_start = oracle.argsort(idx, K)
    assert np.array_equal(perm.cpu().numpy(), ref_perm)
    assert np.array_equal(start.cpu().numpy().astype(np.int64), ref_start)


UPDATE_CASES = [(20000, 128, 100, "bf16", "equal"), (50000, 128, 1000, "bf16", "zipf1.2"),
                (16384, 32, 64, "f32", "equal"), (3001, 64, 300, "bf16", "equal"), (1000, 256, 10, "bf16", "equal"),
                (9000, 8, 20, "f32", "equal"), (200000, 64, 16384, "bf16", "zipf1.2")]


@pytest.mark.parametrize("N,D,K,dtype,weights", UPDATE_CASES)
def test_update_matches_member_means(N, D, K, dtype, weights):
    X, _ = _mixture(N, D, K, dtype, seed=N, weights=weights)
    rng = np.random.default_rng(K)
    if weights.startswith("zipf"):
        w = np.arange(1, K + 1) ** -1.2
        idx = rng.choice(K, N, p=w / w.sum()).astype(np.int32)
    else:
        idx = rng.integers(0, K, N).astype(np.int32)
    idx[:N // 10] = 0  # a hot cluster spanning many blocks
    Cprev = torch.randn(K, D, device=DEV)
    C = Cprev.clone()
    C, counts = km.update(X, torch.from_numpy(idx).to(DEV), C)
    torch.cuda.synchronize()
    Cref, cref = oracle.update(X, idx, Cprev)
    assert np.array_equal(counts.cpu().numpy(), cref)
    assert centroid_rel_err(C, Cref) <= CTOL[dtype]
    empty = cref == 0
    assert torch.equal(C[torch.from_numpy(empty).to(DEV)], Cprev[torch.from_numpy(empty).to(DEV)])


# The fused one-CTA-per-instance update: row sizes of 16 to 512 bytes (one
# to four 128-byte word groups per lane), row stages of one to 32 rows,
# clusters longer than a warp range and single-row clusters.
FUSED = [(5, 4096, 64, 256, "bf16"), (3, 1000, 128, 37, "bf16"), (4, 8192, 32, 1024, "bf16"),
         (2, 3000, 256, 100, "bf16"), (3, 2500, 192, 300, "bf16"), (2, 777, 8, 5, "bf16"),
         (3, 16, 256, 4, "bf16"), (2, 4096, 64, 256, "f32"), (3, 1500, 24, 700, "f32"), (2, 8192, 64, 1024, "f32")]


@pytest.mark.parametrize("B,N,D,K,dtype", FUSED)
def test_update_batched_fused_path(B, N, D, K, dtype):
    X, _ = _mixture(N, D, K, dtype, B=B, seed=B)
    rng = np.random.default_rng(B)
    idx = rng.integers(0, K, (B, N)).astype(np.int32)
    idx[:, : N // 5] = K - 1
    Cprev = torch.randn(B, K, D, device=DEV)
    assert km.plan(km.OP_UPDATE, B, N, D, K, km.BF16 if dtype == "bf16" else km.F32)["update_form"] == 1
    C, counts = km.update(X, torch.from_numpy(idx).to(DEV), Cprev.clone())
    torch.cuda.synchronize()
    for b in range(B):
        Cref, cref = oracle.update(X[b], idx[b], Cprev[b])
        assert np.array_equal(counts[b].cpu().numpy(), cref)
        assert centroid_rel_err(C[b], Cref) <= CTOL[dtype]


def _stepwise(X, C0, iters, kind):
    """Each half of each iteration against the oracle on the inputs it got."""
    dt = torch.bfloat16 if kind == "bf16" else torch.float32
    Cm = C0.float().clone()
    for _ in range(iters):
        Cop = Cm.to(dt)
        idx, md, _ = km.assign(X, Cop)
        check_assignment(X, Cop, idx, md, kind)
        Cref, cref = oracle.update(X, idx.cpu().numpy(), Cm)
        Cm, counts = km.update(X, idx, Cm)
        torch.cuda.synchronize()
        assert np.array_equal(counts.cpu().numpy(), cref)
        assert centroid_rel_err(Cm, Cref) <= CTOL[kind]
    return Cm


def test_stepwise_bf16_several_iterations():
    X, C0 = _mixture(30000, 128, 300, "bf16", seed=11)
    _stepwise(X, C0, 4, "bf16")


def test_stepwise_f32_small_workload():
    wl = WORKLOADS["small_f32"]
    X, C0, _ = make_problem(wl, seed=0, device=DEV)
    _stepwise(X, C0, wl.iters, "f32")


@pytest.mark.parametrize("N,D,K,dtype,iters", [(30000, 128, 300, "bf16", 6), (16384, 32, 64, "f32", 10),
                                               (5000, 64, 1000, "bf16", 3)])
def test_fit_objective_trajectory(N, D, K, dtype, iters):
    """Step-wise: J_t of the fit equals the oracle's exact objective under the
    centroids the fit assigned with at step t (C_{t-1} from a fit of t-1
    iterations, as the operand the tensor cores saw), within 1e-4, for every t.
    Then the fit's whole trajectory against the oracle's own: identical at
    t=1, and within a looser bound at the end (the two trajectories may part
    on an allowed near-tie decision and then re-converge)."""
    X, C0 = _mixture(N, D, K, dtype, seed=5)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    r = km.fit(X, C0, iters)
    torch.cuda.synchronize()
    J = r["objective"].cpu().numpy()
    Cprev = C0
    for t in range(1, iters + 1):
        rt = km.fit(X, C0, t)
        torch.cuda.synchronize()
        assert rt["objective"][t - 1].item() == J[t - 1]  # deterministic: same prefix
        _, d1, _ = oracle.assign(X, Cprev.to(tdt))
        Jref = d1.sum()
        assert abs(J[t - 1] - Jref) <= JTOL * Jref, (t, J[t - 1], Jref)
        Cprev = rt["C"]
    ref = oracle.fit(X, C0, iters, mirror=dtype)
    assert abs(J[0] - ref["J"][0]) <= JTOL * ref["J"][0]
    assert abs(J[-1] - ref["J"][-1]) <= 1e-3 * ref["J"][-1]
    # the final centroids are the member means under the final assignment
    Cchk, cchk = oracle.update(X, r["idx"].cpu().numpy(), r["C"])
    assert np.array_equal(r["counts"].cpu().numpy(), cchk)
    assert centroid_rel_err(r["C"], Cchk) <= CTOL[dtype]


def test_fit_batched_matches_per_instance_oracle():
    B, N, D, K, T = 4, 4096, 64, 256, 5
    X, C0 = _mixture(N, D, K, "bf16", B=B, seed=9, sigma=0.5)
    r = km.fit(X, C0, T)
    rp = km.fit(X, C0, T - 1)
    torch.cuda.synchronize()
    for b in range(B):
        ref = oracle.fit(X[b], C0[b], T, mirror="bf16")
        J = r["objective"][b].cpu().numpy()
        assert abs(J[0] - ref["J"][0]) <= JTOL * ref["J"][0]
        # step-wise last iteration: exact objective under the fit's own C_{T-1}
        _, d1, _ = oracle.assign(X[b], rp["C"][b].to(torch.bfloat16))
        assert abs(J[-1] - d1.sum()) <= JTOL * d1.sum()
        assert abs(J[-1] - ref["J"][-1]) <= 1e-3 * ref["J"][-1]
        Cchk, _ = oracle.update(X[b], r["idx"][b].cpu().numpy(), r["C"][b])
        assert centroid_rel_err(r["C"][b], Cchk) <= CTOL["bf16"]


def test_fit_is_bitwise_deterministic():
    X, C0 = _mixture(200000, 128, 1024, "bf16", seed=2, weights="zipf1.2")
    a = km.fit(X, C0, 3)
    b = km.fit(X, C0, 3)
    torch.cuda.synchronize()
    assert torch.equal(a["C"], b["C"])
    assert torch.equal(a["idx"], b["idx"])
    assert torch.equal(a["objective"], b["objective"])


def test_fit_resume_equals_continuous():
    """Lloyd state is the centroid set: fit(3) then fit(2) from its float32
    centroids equals fit(5) when the operand copy is exact (f32 path)."""
    X, C0 = _mixture(20000, 32, 50, "f32", seed=4)
    full = km.fit(X, C0, 5)
    part = km.fit(X, C0, 3)
    rest = km.fit(X, part["C"].clone(), 2)
    torch.cuda.synchronize()
    assert torch.equal(full["C"], rest["C"])
    assert torch.equal(full["objective"][3:], rest["objective"])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_fit_host_stream_matches_in_core(dtype):
    N, D, K, T = 50000, 128 if dtype == "bf16" else 32, 100, 4
    X, C0 = _mixture(N, D, K, dtype, seed=8)
    Xh = X.cpu().pin_memory()
    ref = km.fit(X, C0, T)
    out = km.fit_host(Xh, C0, T, chunk_rows=12345, want_idx=True)
    torch.cuda.synchronize()
    np.testing.assert_allclose(out["objective"].numpy()[:1], ref["objective"].cpu().numpy()[:1], rtol=JTOL)
    np.testing.assert_allclose(out["objective"].numpy(), ref["objective"].cpu().numpy(), rtol=1e-3)
    oref = oracle.fit(X, C0, T, mirror=dtype)
    np.testing.assert_allclose(out["objective"].numpy()[:1], oref["J"][:1], rtol=JTOL)
    # streamed fit: the final centroids are the member means of its final assignment
    Cchk, _ = oracle.update(X, out["idx"].cpu().numpy(), out["C"])
    assert centroid_rel_err(out["C"], Cchk) <= CTOL[dtype]


def test_edge_k1_gives_global_mean():
    X, C0 = _mixture(10000, 64, 1, "bf16", seed=1)
    r = km.fit(X, C0, 2)
    torch.cuda.synchronize()
    mean = f64(X).mean(0)
    assert centroid_rel_err(r["C"], mean[None]) <= 1e-5
    assert r["counts"].item() == 10000


def test_edge_k_equals_n_identity():
    g = torch.Generator().manual_seed(0)
    X = torch.randint(-8, 9, (300, 16), generator=g).float()
    X = torch.unique(X, dim=0)[:256].contiguous().to(DEV)
    r = km.fit(X.to(torch.bfloat16), X.to(torch.bfloat16), 2)
    torch.cuda.synchronize()
    assert torch.equal(r["idx"].cpu(), torch.arange(X.shape[0], dtype=torch.int32))
    assert float(r["objective"].abs().max()) == 0.0


def test_empty_clusters_keep_previous_centroid():
    X, _ = _mixture(5000, 64, 10, "bf16", seed=6)
    C0 = X[:10].clone()
    C0[7] = 1000.0  # far away: never nearest, stays empty
    r = km.fit(X, C0, 3)
    torch.cuda.synchronize()
    assert r["counts"][7].item() == 0
    assert torch.equal(r["C"][7].cpu(), C0[7].float().cpu())


def test_bounded_wait_timeout_is_reported_and_context_survives():
    assert km.selftest_timeout(2_000_000) == 5  # KM_ERR_TIMEOUT
    X, C = _mixture(1000, 64, 10, "bf16")
    idx, md, _ = km.assign(X, C)
    torch.cuda.synchronize()
    check_assignment(X, C, idx, md, "bf16")


def test_invalid_calls_raise_before_launch():
    X, C = _mixture(1000, 64, 10, "bf16")
    with pytest.raises(km.KMError):
        km.assign(X[:, :60].contiguous(), C[:, :60].contiguous())  # D % 8 != 0 after slicing to 60? 60%8=4
    small = torch.empty(16, dtype=torch.uint8, device=DEV)
    with pytest.raises(ValueError):
        km.assign(X, C, workspace=small)
