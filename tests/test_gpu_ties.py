"""Exact ties inside one 32-column chunk of the assignment epilogue, on
non-integer data.

A point equal to a centroid has distance 0, but the expanded form the tensor
cores accumulate (||x||^2 + ||c||^2 - 2 x.c in float32) lands a few ulps on
either side of 0.  With a duplicated centroid the two scores are
bit-identical, so the tie rule (lowest index wins) must hold for negative
scores too.  Duplicate pairs (k, k+1) sit inside one 32-column chunk (at the
start, the middle and the end of a chunk, at the end of a centroid tile and
of the ragged last tile) and across a chunk edge; the points lying exactly on
them must be assigned to k, bit for bit equal to the oracle, under every
centroid tile width and both kernel forms."""

import numpy as np
import pytest
import torch

import means_clustering_flashassign_b200 as km
import oracle
from synth import WORKLOADS, make_problem
from tests.parity import check_assignment

pytestmark = pytest.mark.gpu

# (k, k+1) pairs: inside a chunk (start, middle, end), at a 256-tile end, at
# the ragged end, and one across a chunk edge (31 | 32 of the second tile)
PAIRS_BF16 = [(0, 1), (5, 6), (30, 31), (81, 82), (254, 255), (287, 288), (511, 512), (597, 598)]
PAIRS_F32 = [(0, 1), (5, 6), (30, 31), (81, 82), (126, 127), (159, 160), (297, 298)]


def _tilings(dtype, D, K):
    """One fitting tiling per (form, centroid tile width)."""
    out = []
    for pair in (0, 1):
        for bn in (64, 128, 256):
            for xb, cs in ((2, 4), (2, 3), (2, 2), (1, 2)):
                t = f"{pair},{bn},{xb},{cs}"
                try:
                    import os
                    os.environ["KM_ASSIGN_TILE"] = t
                    km.plan(km.OP_ASSIGN, 1, 5000, D, K, dtype)
                except km.KMError:
                    continue
                finally:
                    os.environ.pop("KM_ASSIGN_TILE", None)
                out.append(t)
                break
    return out


def _problem(dtype, D, K, pairs, seed):
    wl = WORKLOADS["1m_k1024"].with_(N=5000, D=D, K=K, dtype=dtype,
                                     centers="normal2" if dtype == "bf16" else "uniform10")
    X, C, _ = make_problem(wl, seed=seed, device="cpu")
    C = C.clone()
    X = X.clone()
    on = []
    for j, (k, k1) in enumerate(pairs):
        C[k1] = C[k]
        # eight points exactly on the pair, spread over point tiles
        rows = [j * 8 + r * 613 for r in range(8)]
        X[rows] = C[k]
        on += [(row, k) for row in rows]
    return X.contiguous(), C.contiguous(), on


@pytest.mark.parametrize("dtype,D,K,pairs", [("bf16", 128, 600, PAIRS_BF16), ("f32", 32, 300, PAIRS_F32)])
def test_exact_ties_in_one_chunk_go_to_the_lowest_index(dtype, D, K, pairs, monkeypatch):
    kdt = km.BF16 if dtype == "bf16" else km.F32
    tilings = _tilings(kdt, D, K)
    assert len(tilings) >= (5 if dtype == "bf16" else 2), tilings
    X, C, on = _problem(dtype, D, K, pairs, seed=K)
    rows = np.array([r for r, _ in on])
    want = np.array([k for _, k in on])
    io, _, _ = oracle.assign(X, C)
    assert np.array_equal(io[rows], want)  # the oracle's lowest-index rule
    Xg, Cg = X.cuda(), C.cuda()
    for t in tilings:
        monkeypatch.setenv("KM_ASSIGN_TILE", t)
        idx, md, _ = km.assign(Xg, Cg)
        torch.cuda.synchronize()
        got = idx.cpu().numpy()
        assert np.array_equal(got[rows], want), (t, got[rows][got[rows] != want], want[got[rows] != want])
        assert float(md.cpu()[rows].max()) >= 0.0
        # the duplicates (k+1) never win anywhere
        assert not np.isin(got, [k1 for _, k1 in pairs]).any(), t
        check_assignment(X, C, idx, md, dtype)
