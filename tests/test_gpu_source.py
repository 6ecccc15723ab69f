"""km_fit_source: the out-of-core fit over a point set that is never held
whole in host memory (rows come from a callback, chunk by chunk, every
iteration).  With the same chunking it runs the same kernels on the same
rows as km_fit_host, so the two must agree bit for bit, whether the source
fills two caller-owned staging buffers in turn or points into a pinned pool.
A source that fails (returns unpinned memory, or raises) stops the fit with
an error and leaves the context usable."""

import pytest
import torch

import means_clustering_flashassign_b200 as km
from synth import WORKLOADS, make_problem

pytestmark = pytest.mark.gpu


def _problem(N=50_000, D=128, K=300, dtype="bf16", seed=12):
    wl = WORKLOADS["1m_k1024"].with_(N=N, D=D, K=K, dtype=dtype,
                                     centers="normal2" if dtype == "bf16" else "uniform10")
    X, C0, _ = make_problem(wl, seed=seed, device="cuda")
    return X.contiguous(), C0.contiguous()


def _same(a, b):
    for k in ("C", "counts", "objective"):
        assert torch.equal(torch.as_tensor(a[k]).cpu(), torch.as_tensor(b[k]).cpu()), k
    if a.get("idx") is not None:
        assert torch.equal(a["idx"], b["idx"])


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("f32", 32)])
def test_staging_source_equals_fit_host(dtype, D):
    X, C0 = _problem(D=D, dtype=dtype)
    Xh = X.cpu().pin_memory()
    chunk = 12_345
    ref = km.fit_host(Xh, C0, 3, chunk, want_idx=True)
    stage = [torch.empty((chunk, D), dtype=X.dtype, pin_memory=True) for _ in range(2)]
    calls = []

    def source(row0, rows, slot):
        calls.append((row0, rows, slot))
        stage[slot][:rows].copy_(Xh[row0:row0 + rows])
        return stage[slot][:rows]

    out = km.fit_source(source, X.shape[0], C0, 3, chunk, dtype=X.dtype, want_idx=True)
    _same(out, ref)
    nch = -(-X.shape[0] // chunk)
    assert len(calls) == 3 * nch
    assert [c[2] for c in calls] == [g & 1 for g in range(3 * nch)]
    assert all(r0 == (g % nch) * chunk for g, (r0, _, _) in enumerate(calls))


def test_pool_source_streams_a_larger_set_than_the_pool():
    """Rows i of the streamed set are pool rows i mod P: the fit over two
    copies of the pool equals the fit over the pool itself in its counts
    (doubled) and its centroids (member means, the same points twice)."""
    X, C0 = _problem(N=40_000, K=200)
    P = X.shape[0]
    pool = X.cpu().pin_memory()
    chunk = 10_000  # divides P: every chunk is one slice of the pool

    def source(row0, rows, slot):
        r = row0 % P
        return pool[r:r + rows]

    two = km.fit_source(source, 2 * P, C0, 1, chunk, want_idx=True)
    one = km.fit_host(pool, C0, 1, chunk, want_idx=True)
    assert torch.equal(two["idx"][:P], one["idx"]) and torch.equal(two["idx"][P:], one["idx"])
    assert torch.equal(two["counts"], 2 * one["counts"])
    assert torch.allclose(two["C"], one["C"], rtol=1e-6, atol=1e-6)
    assert abs(float(two["objective"][0]) - 2 * float(one["objective"][0])) <= 1e-9 * float(one["objective"][0])


def test_failing_sources_stop_the_fit_cleanly():
    X, C0 = _problem(N=20_000, K=50)
    Xh = X.cpu().pin_memory()
    ref = km.fit_host(Xh, C0, 2, 5000)

    def unpinned(row0, rows, slot):
        return X.cpu()[row0:row0 + rows]

    with pytest.raises(ValueError, match="pinned"):
        km.fit_source(unpinned, X.shape[0], C0, 2, 5000)

    def broken(row0, rows, slot):
        if row0 >= 10_000:
            raise RuntimeError("storage went away")
        return Xh[row0:row0 + rows]

    with pytest.raises(RuntimeError, match="storage went away"):
        km.fit_source(broken, X.shape[0], C0, 2, 5000)
    _same(km.fit_host(Xh, C0, 2, 5000), ref)
