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

import os

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
                    os.environ["KM_ASSIGN_TILE"] = t
                    km.plan(km.OP_ASSIGN, 1, 5000, D, K, dtype)
                except km.KMError:
                    continue
                finally:
                    os.environ.pop("KM_ASSIGN_TILE", None)
                out.append(t)
                break
    return out


def _problem(dtype, D, K, pairs, seed, B=1):
    wl = WORKLOADS["1m_k1024"].with_(N=5000, D=D, K=K, B=B, dtype=dtype,
                                     centers="normal2" if dtype == "bf16" else "uniform10")
    X, C, _ = make_problem(wl, seed=seed, device="cpu")
    C = C.clone()
    X = X.clone()
    if B > 1:
        return X, C, None
    on = []
    for j, (k, *copies) in enumerate(pairs):
        for k1 in copies:
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
        assert not np.isin(got, [k1 for _, *c in pairs for k1 in c]).any(), t
        check_assignment(X, C, idx, md, dtype)


def test_three_copies_in_one_chunk_and_batched_instances():
    """Three copies of a centroid in one chunk (the lowest is not the
    chunk's first column), and duplicate pairs in each instance of a batch,
    at other columns per instance: every point on a copy takes the lowest
    copy of its own instance."""
    groups = [(200, 204, 217), (40, 63), (3, 31)]
    X, C, on = _problem("bf16", 128, 600, groups, seed=7)
    rows = np.array([r for r, _ in on])
    want = np.array([k for _, k in on])
    for t in _tilings(km.BF16, 128, 600):
        os.environ["KM_ASSIGN_TILE"] = t
        try:
            idx, _, _ = km.assign(X.cuda(), C.cuda())
        finally:
            os.environ.pop("KM_ASSIGN_TILE", None)
        assert np.array_equal(idx.cpu().numpy()[rows], want), t
    B, K = 3, 300
    Xb, Cb, _ = _problem("bf16", 64, K, [], seed=9, B=B)
    want_b = []
    for b in range(B):
        k = 10 + 37 * b
        Cb[b, k + 5] = Cb[b, k]
        Cb[b, k + 9] = Cb[b, k]
        Xb[b, 100 + b] = Cb[b, k]
        Xb[b, 2000 + b] = Cb[b, k]
        want_b.append(k)
    idx, _, _ = km.assign(Xb.cuda().contiguous(), Cb.cuda().contiguous())
    got = idx.cpu().numpy()
    for b in range(B):
        assert got[b, 100 + b] == want_b[b] and got[b, 2000 + b] == want_b[b], (b, got[b, 100 + b], got[b, 2000 + b])
        check_assignment(Xb[b], Cb[b], idx[b], None, "bf16")
