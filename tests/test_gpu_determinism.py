"""Bitwise reproducibility of whole fits on the two-pass sort path.

K = 16,384 clusters need 14-bit keys, so the Sort-Inverse Update sorts in two
radix passes, and a quarter of the points on one spot make one cluster whose
sums cross every segmented-sum block and take the finaliser's whole-block
path.  Every kernel of the iteration chains to the previous one
by programmatic dependent launch.  Ten fits in one process must return the
same centroids, assignment, counts and objective bit for bit; the objective
is summed from per-tile partials in a fixed order, so it does not depend on
how the assignment kernel dealt its tiles to CTAs."""

import numpy as np
import pytest
import torch

import means_clustering_flashassign_b200 as km
from synth import WORKLOADS, make_problem

pytestmark = pytest.mark.gpu


def _zipf_problem(N, K, seed):
    wl = WORKLOADS["4m_k16384_zipf"].with_(N=N, K=K)
    X, C0, _ = make_problem(wl, seed=seed, device="cuda")
    return X.contiguous(), C0.contiguous()


def test_two_pass_zipf_fits_are_bit_identical():
    X, C0 = _zipf_problem(1 << 20, 16384, seed=3)
    # random-point centroids split the Zipf components' points among many
    # clusters; a quarter of the points on one spot makes one hot cluster
    # whose sums cross every segmented-sum block (the finaliser's
    # whole-block path)
    X[::4] = X[0]
    assert km.plan(km.OP_FIT, 1, X.shape[0], 128, 16384, km.BF16)["sort_passes"] == 2
    ref = None
    for _ in range(10):
        r = km.fit(X, C0, 3)
        torch.cuda.synchronize()
        cur = (r["C"].clone(), r["idx"].clone(), r["counts"].clone(), r["objective"].clone())
        if ref is None:
            ref = cur
            continue
        assert torch.equal(cur[0], ref[0])
        assert torch.equal(cur[1], ref[1])
        assert torch.equal(cur[2], ref[2])
        assert torch.equal(cur[3], ref[3])
    # the hot cluster crosses many segmented-sum blocks
    assert int(ref[2].max()) >= X.shape[0] // 4


def test_fit_objective_equals_the_assign_objective_bitwise_up_to_order():
    """J_1 of a fit is the assignment objective under C0: the same per-tile
    partials as km_assign's, reduced in another fixed order, so the two agree
    to rounding and each is stable from call to call."""
    X, C0 = _zipf_problem(300_000, 4096, seed=4)
    fits = [km.fit(X, C0, 1)["objective"][0].item() for _ in range(3)]
    assigns = [km.assign(X, C0, want_mindist=False)[2].item() for _ in range(3)]
    torch.cuda.synchronize()
    assert len(set(fits)) == 1 and len(set(assigns)) == 1
    assert abs(fits[0] - assigns[0]) <= 1e-12 * abs(assigns[0])


@pytest.mark.parametrize("N,K", [(200_000, 5000), (1 << 20, 16384)])
def test_chained_and_plain_order_agree_on_repeated_two_pass_fits(N, K, monkeypatch):
    X, C0 = _zipf_problem(N, K, seed=N % 97)
    monkeypatch.setenv("KM_PDL", "0")
    plain = km.fit(X, C0, 3)
    torch.cuda.synchronize()
    plain = {k: v.clone() for k, v in plain.items()}
    monkeypatch.delenv("KM_PDL")
    for _ in range(3):
        r = km.fit(X, C0, 3)
        torch.cuda.synchronize()
        for k in ("C", "idx", "counts", "objective"):
            assert torch.equal(r[k], plain[k]), k
    assert np.isfinite(plain["objective"].cpu().numpy()).all()
