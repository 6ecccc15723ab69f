"""km_assign_static: the assignment for callers that cannot allocate device
memory (their host framework owns the whole device pool, or cudaMalloc's
synchronisation and cost are not acceptable in their loop).  Its scratch is a
fixed static device array inside libkm.so instead of a caller workspace.

The GPU test calls it through the C ABI twice in a row, on different inputs,
and checks each result against km_assign with a workspace, within the
parity tolerances of the other tests (both run the same kernels, so the
results are expected to be identical).  This file is collected last so that
a failure here cannot hide the other tests' results."""

import ctypes

import numpy as np
import pytest
import torch

import means_clustering_flashassign_b200 as km
from synth import WORKLOADS, make_problem
from tests.parity import JTOL


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


@pytest.mark.gpu
def test_static_scratch_matches_workspace_assign_twice():
    cases = [(WORKLOADS["1m_k1024"].with_(N=300_000, K=1024), 0),
             (WORKLOADS["small_f32"], 1)]
    for wl, seed in cases:  # two calls in a row on different inputs
        X, C, _ = make_problem(wl, seed=seed, device="cuda")
        X, C = X.contiguous(), C.contiguous()
        idx_s, md_s, obj_s = _call_static(X, C, wl.K)
        idx_w, md_w, obj_w = km.assign(X, C)
        torch.cuda.synchronize()
        assert torch.equal(idx_s, idx_w)
        np.testing.assert_allclose(md_s.cpu().numpy(), md_w.cpu().numpy(), rtol=1e-6, atol=1e-6)
        np.testing.assert_allclose(obj_s.cpu().numpy(), obj_w.cpu().numpy(), rtol=JTOL)


def test_oversized_request_is_refused_before_launch():
    L = km.library()
    # 8M points of bf16 D=128 need about 34 MiB of scratch, beyond the 16 MiB area
    st = L.km_assign_static(None, None, 1, 8 << 20, 128, 1024, km.BF16, None, None, None, None)
    assert st == 2  # KM_ERR_UNSUPPORTED
    assert b"static area" in L.km_last_error()
