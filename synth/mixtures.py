"""Gaussian-mixture workloads for exact Lloyd K-Means.

Flash-KMeans (gist.science summary, "研究背景与问题定义" and "实验结果") evaluates on
unnamed workloads; the shapes below are the five synthetic stand-ins this
library is measured on.  Every draw goes through a seeded ``torch.Generator``
so that the same (workload, seed, device) always yields the same tensors.

Recipe per instance:
  * component centres: uniform in [-R, R]^D, or N(0, s^2 I);
  * component weights: equal, or Zipf(s) (w_k proportional to (k+1)^-s);
  * labels: iid categorical draws from the weights (inverse-CDF lookup of
    uniform draws; the CDF is a float64 sum on the CPU);
  * points: centre[label] + sigma * N(0, I) in float32, then cast to the
    workload dtype (bfloat16 casts round to nearest even);
  * initial centroids: rows of X at the first K entries of a seeded random
    permutation of the point indices (so K distinct points).
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    N: int
    D: int
    K: int
    B: int = 1
    dtype: str = "bf16"          # "bf16" or "f32"
    comps: int = 0               # mixture components (default: K)
    centers: str = "normal2"     # "uniform10" or "normal2"
    sigma: float = 1.0
    weights: str = "equal"       # "equal" or "zipf1.2"
    iters: int = 10
    host_resident: bool = False  # X lives in pinned host memory and is streamed
    pool_rows: int = 0           # > 0: the N rows are streamed from a pool of this many rows,
                                 # row i being pool row i mod pool_rows (the set is never held whole)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # N=16384, D=32, K=64 fp32; centres U[-10,10]^D; sigma 1; 10 iterations
    "small_f32": Workload("small_f32", N=16384, D=32, K=64, dtype="f32",
                          centers="uniform10", sigma=1.0, iters=10),
    # N=1M, D=128, K=1024 bf16; centres N(0,4I); sigma 1; 20 iterations
    "1m_k1024": Workload("1m_k1024", N=1 << 20, D=128, K=1024, iters=20),
    # N=4M, D=128, K=16384 bf16; Zipf(1.2) weights (hot clusters); 10 iterations
    "4m_k16384_zipf": Workload("4m_k16384_zipf", N=1 << 22, D=128, K=16384,
                               weights="zipf1.2", iters=10),
    # 512 independent problems of N=4096, D=64, K=256 bf16, sigma 0.5; 25 iterations
    "batch512_k256": Workload("batch512_k256", N=4096, D=64, K=256, B=512,
                              sigma=0.5, iters=25),
    # N=268M, D=128, K=4096 bf16 in pinned host memory, streamed in 16M-row chunks
    "ooc_268m_k4096": Workload("ooc_268m_k4096", N=1 << 28, D=128, K=4096,
                               iters=5, host_resident=True),
    # N=2^30 (one billion) rows, D=128, K=4096 bf16: 256 GiB, never held
    # whole; streamed in 16M-row chunks from a 2^28-row pinned pool (the
    # ooc_268m_k4096 points), row i = pool row i mod 2^28
    "ooc_1b_k4096": Workload("ooc_1b_k4096", N=1 << 30, D=128, K=4096,
                             iters=3, host_resident=True, pool_rows=1 << 28),
}


def instance_seed(seed: int, b: int) -> int:
    """Seed of instance b of a batched workload."""
    return (int(seed) * 1_000_003 + int(b) * 7919 + 17) & ((1 << 62) - 1)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _mixture(wl: Workload, seed: int, device):
    """Generator, component centres and the cumulative component weights.

    The cumulative weights are formed on the CPU in float64 (a fixed
    sequential sum) and labels are drawn by inverse-CDF lookup of uniform
    draws: a device cumulative sum (as inside a CUDA multinomial) may
    associate its float additions differently from run to run, which moves
    labels at bucket edges and makes the same seed give different points."""
    comps = wl.comps or wl.K
    g = _gen(seed, device)
    if wl.centers == "uniform10":
        mu = (torch.rand(comps, wl.D, generator=g, device=device) * 20.0 - 10.0)
    elif wl.centers == "normal2":
        mu = torch.randn(comps, wl.D, generator=g, device=device) * 2.0
    else:
        raise ValueError(wl.centers)
    if wl.weights == "equal":
        w = torch.ones(comps, dtype=torch.float64)
    elif wl.weights.startswith("zipf"):
        s = float(wl.weights[4:])
        w = torch.arange(1, comps + 1, dtype=torch.float64).pow(-s)
    else:
        raise ValueError(wl.weights)
    cdf = torch.cumsum(w, 0)
    cdf = (cdf / cdf[-1]).to(torch.float32).to(device)
    return g, mu.float(), cdf


def make_points(wl: Workload, seed: int = 0, device="cpu", rows: Optional[slice] = None,
                out: Optional[torch.Tensor] = None, chunk: int = 1 << 22):
    """Draw the N x D points of one instance (float32 draws cast to the dtype).

    Points are drawn chunk by chunk; chunk c uses its own generator seeded from
    (seed, c), so any row range can be regenerated independently.
    ``out`` (optional) receives the rows (any device, e.g. pinned host memory).
    Returns (X, labels) where labels are the generating components (int64),
    or (out, None) when ``out`` is given.
    """
    g, mu, cdf = _mixture(wl, seed, device)
    start = 0 if rows is None else rows.start
    stop = wl.N if rows is None else rows.stop
    n = stop - start
    X = out if out is not None else torch.empty(n, wl.D, dtype=wl.torch_dtype, device=device)
    labels_all = None if out is not None else torch.empty(n, dtype=torch.int64, device=device)
    c0 = start // chunk
    c1 = (stop + chunk - 1) // chunk
    for c in range(c0, c1):
        lo, hi = c * chunk, min((c + 1) * chunk, wl.N)
        gc = _gen(instance_seed(seed, 1_000_000 + c), device)
        u = torch.rand(hi - lo, generator=gc, device=device)
        lab = torch.searchsorted(cdf, u, right=True).clamp_(max=cdf.numel() - 1)
        pts = mu[lab] + wl.sigma * torch.randn(hi - lo, wl.D, generator=gc, device=device)
        a, b_ = max(lo, start), min(hi, stop)
        piece = pts[a - lo:b_ - lo].to(wl.torch_dtype)
        X[a - start:b_ - start].copy_(piece, non_blocking=False)
        if labels_all is not None:
            labels_all[a - start:b_ - start] = lab[a - lo:b_ - lo]
    return X, labels_all


def init_rows(wl: Workload, seed: int = 0, device="cpu") -> torch.Tensor:
    """Indices of the K initial centroids: first K of a seeded permutation of N
    (of the pool's rows for a pooled workload, so the K rows are distinct)."""
    g = _gen(instance_seed(seed, 999_999), device)
    n = wl.pool_rows if wl.pool_rows else wl.N
    return torch.randperm(n, generator=g, device=device)[: wl.K]


def pool_workload(wl: Workload) -> Workload:
    """The workload whose points form the pool of a pooled workload."""
    return wl.with_(N=wl.pool_rows, pool_rows=0) if wl.pool_rows else wl


def make_problem(wl: Workload, seed: int = 0, device="cpu"):
    """Return (X, C0, labels) for a workload.

    X: (N, D) for B == 1, else (B, N, D); C0 likewise (K, D) / (B, K, D),
    taken as exact copies of rows of X.  labels: generating components.
    """
    if wl.B == 1:
        X, lab = make_points(wl, seed, device)
        sel = init_rows(wl, seed, device)
        return X, X[sel].clone(), lab
    Xs, Cs, Ls = [], [], []
    for b in range(wl.B):
        s = instance_seed(seed, b)
        X, lab = make_points(wl, s, device)
        sel = init_rows(wl, s, device)
        Xs.append(X)
        Cs.append(X[sel].clone())
        Ls.append(lab)
    return torch.stack(Xs), torch.stack(Cs), torch.stack(Ls)
