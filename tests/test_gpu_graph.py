"""The fit captured as a CUDA graph (km_fit_graph_*): its launches give
km_fit's results bit for bit, start again from C0 every time, follow new
contents of the argument buffers, time their iterations, count their
kernels at launch, and a failing capture leaves nothing behind."""

import pytest
import torch

import means_clustering_flashassign_b200 as km
from synth import WORKLOADS, make_problem

pytestmark = pytest.mark.gpu

# one instance (CTA pairs), the f32 three-product path, batched (fused update)
CASES = [("bf16", 1, 20000, 128, 300), ("f32", 1, 16384, 32, 64), ("bf16", 8, 4096, 64, 256)]


def _problem(dtype, B, N, D, K, seed):
    wl = WORKLOADS["1m_k1024"].with_(N=N, D=D, K=K, B=B, dtype=dtype,
                                     centers="normal2" if dtype == "bf16" else "uniform10")
    X, C0, _ = make_problem(wl, seed=seed, device="cuda")
    return X.contiguous(), C0.contiguous()


@pytest.mark.parametrize("dtype,B,N,D,K", CASES)
def test_graph_launch_equals_fit(dtype, B, N, D, K):
    X, C0 = _problem(dtype, B, N, D, K, seed=3)
    ref = km.fit(X, C0, 4)
    g = km.FitGraph(X, C0, 4)
    for _ in range(2):  # every launch starts again from C0
        out = g.launch()
        torch.cuda.synchronize()
        for k in ("C", "idx", "counts", "objective"):
            assert torch.equal(out[k], ref[k]), k
    g.close()


def test_graph_follows_buffer_contents():
    X, C0 = _problem("bf16", 1, 10000, 64, 100, seed=4)
    X2, C2 = _problem("bf16", 1, 10000, 64, 100, seed=5)
    g = km.FitGraph(X, C0, 3)
    X.copy_(X2)
    C0.copy_(C2)
    out = g.launch()
    torch.cuda.synchronize()
    ref = km.fit(X2, C2, 3)
    for k in ("C", "idx", "counts", "objective"):
        assert torch.equal(out[k], ref[k]), k
    g.close()


def test_graph_timing_and_launch_count():
    X, C0 = _problem("f32", 1, 16384, 32, 64, seed=6)
    n0 = km.launch_count()
    g = km.FitGraph(X, C0, 10, timed=True)
    assert km.launch_count() == n0  # creation enqueues nothing
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g.launch(stream=s)
    ms = g.iters_ms()
    assert 0 < ms < 1000
    per_launch = km.launch_count() - n0
    n1 = km.launch_count()
    km.fit(X, C0, 10)
    torch.cuda.synchronize()
    assert per_launch == km.launch_count() - n1  # the kernels km_fit enqueues
    g.close()


def test_graph_errors():
    X, C0 = _problem("bf16", 1, 1000, 64, 10, seed=7)
    g = km.FitGraph(X, C0, 2)
    with pytest.raises(km.KMError):
        g.iters_ms()  # created without timing
    g.close()
    gt = km.FitGraph(X, C0, 2, timed=True)
    with pytest.raises(km.KMError):
        gt.iters_ms()  # not launched yet
    gt.close()
    # a call km_fit refuses fails inside the capture; the graph is not made
    # and the library keeps working
    Cbig = torch.zeros(2000, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(km.KMError):
        km.FitGraph(X, Cbig, 2)
    r = km.fit(X, C0, 2)
    torch.cuda.synchronize()
    assert int(r["counts"].sum()) == 1000
