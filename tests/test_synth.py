"""Seeded generators: same seed -> same tensors; shapes, dtypes and init rule."""

import torch

from synth import WORKLOADS, make_problem, make_points, init_rows


def test_deterministic_and_shapes():
    wl = WORKLOADS["small_f32"].with_(N=3000)
    X1, C1, L1 = make_problem(wl, seed=0)
    X2, C2, L2 = make_problem(wl, seed=0)
    assert torch.equal(X1, X2) and torch.equal(C1, C2) and torch.equal(L1, L2)
    assert X1.shape == (3000, 32) and X1.dtype == torch.float32
    assert C1.shape == (64, 32)
    X3, _, _ = make_problem(wl, seed=1)
    assert not torch.equal(X1, X3)


def test_init_rows_are_distinct_points_of_x():
    wl = WORKLOADS["1m_k1024"].with_(N=5000, K=300)
    X, C, _ = make_problem(wl, seed=3)
    sel = init_rows(wl, seed=3)
    assert len(set(sel.tolist())) == 300
    assert torch.equal(C, X[sel])
    assert X.dtype == torch.bfloat16


def test_row_ranges_regenerate_identically():
    wl = WORKLOADS["1m_k1024"].with_(N=10000, K=16)
    X, _ = make_points(wl, seed=0, chunk=4096)
    part = torch.empty(3000, wl.D, dtype=wl.torch_dtype)
    make_points(wl, seed=0, rows=slice(3500, 6500), out=part, chunk=4096)
    assert torch.equal(part, X[3500:6500])


def test_batched_instances_differ():
    wl = WORKLOADS["batch512_k256"].with_(B=3, N=512, K=16)
    X, C, _ = make_problem(wl, seed=0)
    assert X.shape == (3, 512, 64) and C.shape == (3, 16, 64)
    assert not torch.equal(X[0], X[1])


def test_zipf_weights_concentrate():
    wl = WORKLOADS["4m_k16384_zipf"].with_(N=200000, K=1000)
    _, lab = make_points(wl, seed=0)
    top = torch.bincount(lab, minlength=1000).max().item()
    assert top > 0.1 * wl.N


def test_cdf_is_a_fixed_float64_sum():
    """Labels come from a CPU float64 cumulative sum of the weights, so the
    same seed gives the same labels on every run (a device cumulative sum may
    associate its additions differently from run to run)."""
    wl = WORKLOADS["4m_k16384_zipf"].with_(N=50_000)
    _, lab1 = make_points(wl, seed=4)
    _, lab2 = make_points(wl, seed=4)
    assert torch.equal(lab1, lab2)
    assert int(lab1.max()) < wl.K and int(lab1.min()) >= 0


GEN_CHILD = r"""
import hashlib, sys, torch
from synth import WORKLOADS, make_problem
X, C0, L = make_problem(WORKLOADS[sys.argv[1]], seed=0, device="cuda")
h = hashlib.sha256()
for t in (X, C0, L):
    h.update(t.cpu().contiguous().view(torch.uint8).numpy().tobytes())
print(h.hexdigest())
"""


import pytest  # noqa: E402


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["4m_k16384_zipf", "1m_k1024"])
def test_device_generation_is_the_same_in_every_process(name):
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    hashes = {subprocess.run([sys.executable, "-c", GEN_CHILD, name], cwd=root, capture_output=True, text=True,
                             check=True, env=dict(os.environ, PYTHONPATH=root)).stdout.strip() for _ in range(3)}
    assert len(hashes) == 1, hashes
