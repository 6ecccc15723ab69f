"""km_assign_static: the assignment for callers that cannot allocate device
memory (their host framework owns the whole device pool, or cudaMalloc's
synchronisation and cost are not acceptable in their loop).  Its scratch is a
fixed static device array inside libkm.so instead of a caller workspace.

The GPU tests call it through the C ABI twice in a row, on different inputs,
and check each result against km_assign with a workspace, within the
parity tolerances of the other tests (both run the same kernels, so the
results are expected to be identical); one of them runs the largest shape
the array holds.  The CPU test pins the refusal boundary: the shape whose
km_assign workspace is exactly the array's size is accepted, one point more
is refused.  This file is collected last so that a failure here cannot hide
the other tests' results."""

import ctypes

import numpy as np
import pytest
import torch

import means_clustering_flashassign_b200 as km
from synth import WORKLOADS, make_problem
from tests.parity import JTOL

LIMIT = 16 << 20  # KM_ASSIGN_STATIC_SCRATCH_BYTES


def _largest_n(K=1024, D=128, dt=km.BF16):
    """Largest N whose km_assign workspace fits the static area (the
    workspace grows with N: 32 bytes of norm row per point plus the
    objective partials, rounded to 256 bytes)."""
    lo, hi = K, 1 << 22
    while hi - lo > 1:
        m = (lo + hi) // 2
        if km.workspace_size(km.OP_ASSIGN, 1, m, D, K, dt) <= LIMIT:
            lo = m
        else:
            hi = m
    return lo


def _call_static(X, C, K):
    L = km.library()
    B, N, D = (1, *X.shape) if X.dim() == 2 else X.shape
    idx = torch.empty(X.shape[:-1], dtype=torch.int32, device=X.device)
    md = torch.empty(X.shape[:-1], dtype=torch.float32, device=X.device)
    obj = torch.empty(B, dtype=torch.float64, device=X.device)
    dt = km.BF16 if X.dtype == torch.bfloat16 else km.F32
    st = L.km_assign_static(ctypes.c_void_p(X.data_ptr()), ctypes.c_void_p(C.data_ptr()), B, N, D, K, dt,
                            ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(md.data_ptr()),
                            ctypes.c_void_p(obj.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, L.km_last_error()
    return idx, md, obj


def _same_as_workspace_assign(wl, seed):
    X, C, _ = make_problem(wl, seed=seed, device="cuda")
    X, C = X.contiguous(), C.contiguous()
    idx_s, md_s, obj_s = _call_static(X, C, wl.K)
    idx_w, md_w, obj_w = km.assign(X, C)
    torch.cuda.synchronize()
    assert torch.equal(idx_s, idx_w)
    np.testing.assert_allclose(md_s.cpu().numpy(), md_w.cpu().numpy(), rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(obj_s.cpu().numpy(), obj_w.cpu().numpy(), rtol=JTOL)


@pytest.mark.gpu
def test_static_scratch_matches_workspace_assign_twice():
    cases = [(WORKLOADS["1m_k1024"].with_(N=300_000, K=1024), 0),
             (WORKLOADS["small_f32"], 1)]
    for wl, seed in cases:  # two calls in a row on different inputs
        _same_as_workspace_assign(wl, seed)


@pytest.mark.gpu
def test_static_scratch_largest_shape_twice():
    n = _largest_n()
    for seed in (2, 3):
        _same_as_workspace_assign(WORKLOADS["1m_k1024"].with_(N=n, K=1024), seed)


def test_refusal_boundary_is_the_static_size():
    L = km.library()
    n = _largest_n()
    assert km.workspace_size(km.OP_ASSIGN, 1, n, 128, 1024, km.BF16) <= LIMIT
    assert km.workspace_size(km.OP_ASSIGN, 1, n + 1, 128, 1024, km.BF16) > LIMIT
    # one point beyond the area: refused on the size, before any device call
    st = L.km_assign_static(None, None, 1, n + 1, 128, 1024, km.BF16, None, None, None, None)
    assert st == 2  # KM_ERR_UNSUPPORTED
    assert b"static area" in L.km_last_error()
    # the largest shape passes the size check (it then fails only on the null
    # pointers or, without a GPU, on the device query)
    st = L.km_assign_static(None, None, 1, n, 128, 1024, km.BF16, None, None, None, None)
    assert st != 2
    # 8M points of bf16 at D=128 need about 258 MiB (32 bytes of norm row per
    # point): far beyond the 16 MiB area
    st = L.km_assign_static(None, None, 1, 8 << 20, 128, 1024, km.BF16, None, None, None, None)
    assert st == 2
