"""The two baselines the method replaces (materialised distances, atomic
scatter update), built for measurement only, against the same oracle rules
as the method itself."""

import numpy as np
import pytest
import torch

import means_clustering_flashassign_b200 as km
import oracle
from synth import WORKLOADS, make_problem
from tests.parity import CTOL, centroid_rel_err, check_assignment

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _mixture(N, D, K, dtype, seed):
    wl = WORKLOADS["1m_k1024"].with_(N=N, D=D, K=K, dtype=dtype,
                                     centers="normal2" if dtype == "bf16" else "uniform10")
    X, C0, _ = make_problem(wl, seed=seed, device=DEV)
    return X.contiguous(), C0.contiguous()


@pytest.mark.parametrize("N,D,K,dtype,chunk", [(5000, 128, 300, "bf16", 1536), (3001, 64, 257, "bf16", None),
                                               (4000, 32, 100, "f32", 999)])
def test_materialised_assign_matches_oracle(N, D, K, dtype, chunk):
    X, C = _mixture(N, D, K, dtype, seed=N + K)
    idx, md = km.ablation_assign_materialized(X, C, chunk_rows=chunk)
    torch.cuda.synchronize()
    check_assignment(X, C, idx, md, dtype)


def test_materialised_assign_integer_data_exact_with_ties():
    g = torch.Generator().manual_seed(9)
    X = torch.randint(-3, 4, (2500, 64), generator=g).to(torch.bfloat16)
    C = torch.randint(-3, 4, (300, 64), generator=g).to(torch.bfloat16)
    C[150:200] = C[0:50]
    X[:40] = C[:40]
    idx, md = km.ablation_assign_materialized(X.to(DEV), C.to(DEV), chunk_rows=1000)
    io, d1, _ = oracle.assign(X, C)
    assert np.array_equal(idx.cpu().numpy(), io)
    assert np.array_equal(md.cpu().double().numpy(), d1)


@pytest.mark.parametrize("N,D,K,dtype,weights", [(20000, 128, 512, "bf16", "equal"),
                                                 (20000, 64, 256, "bf16", "zipf1.2"),
                                                 (8000, 32, 64, "f32", "equal")])
def test_atomic_update_matches_member_means(N, D, K, dtype, weights):
    wl = WORKLOADS["1m_k1024"].with_(N=N, D=D, K=K, dtype=dtype, weights=weights,
                                     centers="normal2" if dtype == "bf16" else "uniform10")
    X, C0, _ = make_problem(wl, seed=4, device=DEV)
    idx, _, _ = km.assign(X.contiguous(), C0.contiguous())
    C = C0.float().clone()
    counts = km.ablation_update_atomic(X.contiguous(), idx, C)
    torch.cuda.synchronize()
    Cref, cref = oracle.update(X, idx.cpu().numpy(), C0.float())
    assert np.array_equal(counts.cpu().numpy(), cref)
    assert centroid_rel_err(C, Cref) <= CTOL[dtype]
