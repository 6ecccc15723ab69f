"""Parity helpers shared by the GPU tests: compare CUDA results with the CPU
oracle under the rules the tolerances come from.

Assignment rule (floating point decides an integer): a point whose oracle
best-vs-second gap exceeds rel * (||x||^2 + ||c_best||^2) must get exactly the
oracle's cluster; any other point may take a near-tied centroid, whose exact
distance must then be within that same threshold of the best.  rel is 1e-3
for bfloat16 operands and 1e-6 for float32 operands (TF32 split).
Centroids: max_k ||c_k - c_k^ref||_inf / max(||c_k^ref||_inf, 1e-6) within
1e-3 (bf16) / 1e-5 (f32).  Objective: relative 1e-4.
"""

import numpy as np
import torch

import oracle

GAP = {"bf16": 1e-3, "f32": 1e-6}
CTOL = {"bf16": 1e-3, "f32": 1e-5}
JTOL = 1e-4


def f64(t):
    return t.detach().to("cpu").double().numpy() if hasattr(t, "detach") else np.asarray(t, np.float64)


def check_assignment(X, C, idx_gpu, mindist_gpu=None, kind="bf16", rows=None):
    """X, C: the exact operand values (torch or numpy); idx_gpu: int array."""
    Xd, Cd = f64(X), f64(C)
    if rows is not None:
        Xd = Xd[rows]
    ig = np.asarray(idx_gpu.detach().cpu().numpy() if hasattr(idx_gpu, "detach") else idx_gpu).astype(np.int64)
    if rows is not None and ig.shape[0] != Xd.shape[0]:
        ig = ig[rows]
    assert ig.min() >= 0 and ig.max() < Cd.shape[0]
    io, d1, d2 = oracle.assign(Xd, Cd)
    xn = (Xd * Xd).sum(1)
    cn = (Cd * Cd).sum(1)
    thr = GAP[kind] * (xn + cn[io])
    clear = (d2 - d1) > thr
    bad = np.nonzero(clear & (ig != io))[0]
    assert bad.size == 0, f"{bad.size} clear-gap points disagree, e.g. row {bad[:5]}"
    dg = ((Xd - Cd[ig]) ** 2).sum(1)
    worst = np.max(dg - d1 - thr)
    assert worst <= 0, f"a near-tie choice is {worst} beyond the threshold"
    if mindist_gpu is not None:
        md = f64(mindist_gpu)
        if rows is not None and md.shape[0] != Xd.shape[0]:
            md = md[rows]
        # fp32 expanded-form distance of the chosen centroid
        err = np.abs(md - dg)
        lim = 1e-5 * (xn + cn[ig]) + 1e-6
        assert np.all(err <= lim), f"mindist off by {np.max(err - lim)} beyond the limit"
    # objective bound: relative JTOL plus the fp32 cancellation floor of the
    # expanded form, summed over points (it matters only when J is ~0)
    jfloor = float((1e-6 * (xn + cn[ig])).sum())
    return dict(n_clear=int(clear.sum()), n=int(clear.size), d1=d1, jfloor=jfloor)


def centroid_rel_err(C_gpu, C_ref):
    Cg, Cr = f64(C_gpu), f64(C_ref)
    scale = np.maximum(np.abs(Cr).max(1), 1e-6)
    return float(np.max(np.abs(Cg - Cr).max(1) / scale))


def bf16_round(t):
    return t.to(torch.bfloat16)
