"""Seeded random shapes: one Lloyd iteration of the fit entry point on many
small problems (both dtypes, single and batched, ragged N / K / D, every
kernel form the tiling chooser picks for them) against the oracle's
definition of the step: the assignment under C0 by the parity gap rule, the
counts as its histogram, the centroids as the member means of the device's
own assignment (previous centroid for empty clusters) and J_1 as the
objective under C0."""

import numpy as np
import pytest
import torch

import means_clustering_flashassign_b200 as km
import oracle
from synth import WORKLOADS, make_problem
from tests.parity import CTOL, JTOL, centroid_rel_err, check_assignment

pytestmark = pytest.mark.gpu


def _shapes(count, seed):
    rng = np.random.default_rng(seed)
    out = []
    while len(out) < count:
        dtype = "bf16" if rng.random() < 0.7 else "f32"
        D = int(rng.choice([8, 16, 24, 32, 40, 64, 96, 128, 192, 256] if dtype == "bf16" else [8, 16, 24, 32, 40, 64]))
        B = int(rng.choice([1, 1, 1, 2, 3]))
        N = int(rng.integers(1, 6000))
        K = int(rng.integers(1, min(N, 700) + 1))
        out.append((dtype, B, N, D, K, int(rng.integers(0, 1 << 30))))
    return out


@pytest.mark.parametrize("dtype,B,N,D,K,seed", _shapes(64, 2026))
def test_one_iteration_on_random_shapes(dtype, B, N, D, K, seed):
    wl = WORKLOADS["1m_k1024"].with_(N=N, D=D, K=K, B=B, dtype=dtype,
                                     centers="normal2" if dtype == "bf16" else "uniform10")
    X, C0, _ = make_problem(wl, seed=seed, device="cuda")
    X, C0 = X.contiguous(), C0.contiguous()
    r = km.fit(X, C0, 1)
    torch.cuda.synchronize()
    Xs = X if B > 1 else X[None]
    C0s = C0 if B > 1 else C0[None]
    idx = r["idx"].cpu().numpy().reshape(B, N)
    counts = r["counts"].cpu().numpy().reshape(B, K)
    C1 = r["C"].cpu().reshape(B, K, D)
    J = r["objective"].cpu().numpy().reshape(B, -1)
    for b in range(B):
        res = check_assignment(Xs[b].cpu(), C0s[b].cpu(), idx[b], None, dtype)
        assert np.array_equal(counts[b], np.bincount(idx[b], minlength=K))
        Cref, cref = oracle.update(Xs[b].cpu(), idx[b].astype(np.int32), C0s[b].cpu().float())
        assert np.array_equal(counts[b], cref)
        assert centroid_rel_err(C1[b], Cref) <= CTOL[dtype]
        J1 = res["d1"].sum()
        assert abs(float(J[b, 0]) - J1) <= JTOL * J1 + res["jfloor"]
