"""Pins for the CPU oracle (no GPU).

The oracle restates exact Lloyd K-Means ("Flash-KMeans: Fast and
Memory-Efficient Exact K-Means", §2 Methodology: the mathematics is standard
Lloyd, unchanged and without approximation).  These tests pin it to things
other than itself: hand-derived worked examples (tests/golden), closed forms,
independent library routines (scipy's cdist, numpy's stable argsort, torch's
bfloat16 cast, scikit-learn's Lloyd), invariants, and exhaustive brute force
on tiny integer inputs.  ``test_planted_mistakes_are_caught`` compiles copies
of the oracle with plausible mistakes and checks that some pin fails for each.
"""

import itertools
import json
import os
import tempfile

import numpy as np
import pytest
import torch
from scipy.spatial.distance import cdist

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- pin checks
# Each check raises AssertionError when the oracle disagrees with its pin.

def check_golden_1d():
    g = _golden("lloyd_1d_hand.json")
    X, C = np.array(g["X"]), np.array(g["C0"])
    for it in g["iterations"]:
        idx, d1, _ = oracle.assign(X, C)
        assert idx.tolist() == it["idx"]
        assert abs(oracle.objective(d1) - it["J"]) <= 1e-12 * max(1.0, it["J"])
        C, counts = oracle.update(X, idx, C)
        np.testing.assert_allclose(C, np.array(it["C_after"]), rtol=1e-15, atol=0)
        assert counts.tolist() == it["counts"]
    r = oracle.fit(X, np.array(g["C0"]), len(g["iterations"]))
    np.testing.assert_allclose(r["J"], [it["J"] for it in g["iterations"]], rtol=1e-15)


def check_golden_tie():
    g = _golden("tie_duplicate_centroid.json")
    X, C0 = np.array(g["X"]), np.array(g["C0"])
    idx, d1, _ = oracle.assign(X, C0)
    assert idx.tolist() == g["idx"]
    assert d1.tolist() == g["d1"]
    assert oracle.objective(d1) == g["J"]
    C, counts = oracle.update(X, idx, C0)
    assert C.tolist() == g["C_after"]
    assert counts.tolist() == g["counts"]


def check_assign_vs_cdist(seed=0):
    """Argmin and best/second distances against scipy's cdist (float64)."""
    rng = np.random.default_rng(seed)
    for N, D, K in [(300, 7, 13), (257, 33, 1), (64, 2, 64), (500, 16, 40)]:
        X = rng.normal(size=(N, D))
        C = rng.normal(size=(K, D)) * 1.5
        idx, d1, d2 = oracle.assign(X, C)
        Dm = cdist(X, C, "sqeuclidean")
        assert np.array_equal(idx, np.argmin(Dm, axis=1))
        np.testing.assert_allclose(d1, Dm.min(1), rtol=1e-12, atol=1e-12)
        if K > 1:
            np.testing.assert_allclose(d2, np.partition(Dm, 1, axis=1)[:, 1], rtol=1e-12, atol=1e-12)
        else:
            assert np.all(np.isinf(d2))


def check_bruteforce_integer():
    """Exhaustive: every 1-D integer dataset of 4 points in [0,3] against every
    pair of integer centroids; distances are exact integers, so the argmin
    (lowest index on ties), the mean and the objective are checked exactly."""
    vals = range(4)
    for pts in itertools.product(vals, repeat=4):
        X = np.array(pts, dtype=np.float64)[:, None]
        for c0, c1 in itertools.product(vals, repeat=2):
            C = np.array([[c0], [c1]], dtype=np.float64)
            idx, d1, _ = oracle.assign(X, C)
            for i, x in enumerate(pts):
                da, db = (x - c0) ** 2, (x - c1) ** 2
                assert idx[i] == (1 if db < da else 0)
                assert d1[i] == min(da, db)
            Cn, counts = oracle.update(X, idx, C)
            for k in range(2):
                mem = [x for x, a in zip(pts, idx) if a == k]
                assert counts[k] == len(mem)
                assert Cn[k, 0] == (sum(mem) / len(mem) if mem else C[k, 0])


def check_closed_forms(seed=1):
    rng = np.random.default_rng(seed)
    X = rng.normal(size=(1000, 9)) * 3 + 2
    # K = 1: the centroid is the global mean, J is the total squared deviation
    r = oracle.fit(X, X[:1], 2)
    np.testing.assert_allclose(r["C"][0], X.mean(0), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(r["J"][1], X.shape[0] * X.var(0).sum(), rtol=1e-10)
    assert r["counts"].tolist() == [1000]
    # K = N, C0 = X (distinct points): identity assignment, zero objective
    Y = rng.normal(size=(50, 4))
    r = oracle.fit(Y, Y, 3)
    assert r["idx"].tolist() == list(range(50))
    assert np.all(r["J"] == 0.0)
    np.testing.assert_array_equal(r["C"], Y)


def check_separated_mixture(seed=2):
    """Well separated mixture started at the true centres: labels are the
    generating components and the centroids become their sample means."""
    rng = np.random.default_rng(seed)
    K, D, n = 8, 5, 200
    mu = np.arange(K)[:, None] * 100.0 * np.ones((1, D))
    lab = np.repeat(np.arange(K), n)
    rng.shuffle(lab)
    X = mu[lab] + rng.normal(size=(K * n, D)) * 0.1
    r = oracle.fit(X, mu, 2)
    assert np.array_equal(r["idx"], lab)
    for k in range(K):
        np.testing.assert_allclose(r["C"][k], X[lab == k].mean(0), rtol=1e-13, atol=1e-13)


def check_invariants_and_sklearn(seed=3):
    rng = np.random.default_rng(seed)
    X = np.concatenate([rng.normal(loc=m, size=(300, 6)) for m in (-6, 0, 6, 12)])
    C0 = X[rng.permutation(len(X))[:4]]
    T = 8
    r = oracle.fit(X, C0, T)
    # objective never increases in exact float64 Lloyd
    assert np.all(np.diff(r["J"]) <= 1e-9 * r["J"][0])
    # final centroids are the means of their members under the last assignment
    for k in range(4):
        m = r["idx"] == k
        if m.any():
            np.testing.assert_allclose(r["C"][k], X[m].mean(0), rtol=1e-12, atol=1e-12)
    # scikit-learn's Lloyd from the same start agrees (no cluster empties here)
    from sklearn.cluster import KMeans
    km = KMeans(n_clusters=4, init=C0, n_init=1, max_iter=T, tol=0.0, algorithm="lloyd").fit(X)
    # sklearn reports the labels/inertia of its final centroids; compare centroids
    np.testing.assert_allclose(np.sort(r["C"], axis=0), np.sort(km.cluster_centers_, axis=0),
                               rtol=1e-9, atol=1e-9)


def check_bf16_rounding():
    # hand cases: halfway points round to even, just-above rounds up
    cases = {1 + 2**-8: 1.0, 1 + 3 * 2**-8: 1 + 2**-6, 1 + 2**-8 + 2**-30: 1 + 2**-7,
             -(1 + 2**-8): -1.0, 255.5: 256.0, 2.0**-130: 2.0**-130,
             3 * 2.0**-134: 2.0**-132, 0.0: 0.0}
    for v, want in cases.items():
        assert oracle.round_bf16([v])[0] == want, (v, oracle.round_bf16([v])[0], want)
    # agree with torch's float32 -> bfloat16 cast (round to nearest even) on
    # float32-representable inputs, where no double rounding can occur
    rng = np.random.default_rng(4)
    a = np.concatenate([rng.normal(size=5000) * 10.0 ** rng.integers(-30, 30, 5000),
                        rng.normal(size=1000)]).astype(np.float32).astype(np.float64)
    want = torch.from_numpy(a).float().to(torch.bfloat16).double().numpy()
    assert np.array_equal(oracle.round_bf16(a), want)


def check_f32_rounding(seed=7):
    """float32 round-to-nearest-even of doubles (the oracle's f32 mirror mode)
    against numpy's float32 cast, bit for bit, and hand cases derived from the
    format: 23 stored mantissa bits, subnormal spacing 2^-149, largest finite
    value (2 - 2^-23) * 2^127."""
    cases = {1 + 2**-24: 1.0,                      # halfway, ties to even (down)
             1 + 3 * 2**-24: 1 + 2**-22,           # halfway, ties to even (up)
             1 + 2**-24 + 2**-40: 1 + 2**-23,      # just above halfway
             -(1 + 3 * 2**-24): -(1 + 2**-22),
             2.0**-150: 0.0,                       # half the smallest subnormal
             3 * 2.0**-150: 2.0**-148,             # subnormal halfway, to even
             2.0**-149: 2.0**-149,
             (2 - 2**-24) * 2.0**127: np.inf,      # halfway above the largest finite
             (2 - 2**-24 - 2**-40) * 2.0**127: (2 - 2**-23) * 2.0**127,
             0.1: 0.100000001490116119384765625, 0.0: 0.0}
    for v, want in cases.items():
        got = oracle.round_f32([v])[0]
        assert got == want, (v, got, want)
    rng = np.random.default_rng(seed)
    a = np.concatenate([rng.normal(size=20000) * 10.0 ** rng.integers(-45, 39, 20000),
                        rng.normal(size=2000),
                        # exact float32 halfway points: a float32 value plus half its ulp
                        (lambda f: f + np.spacing(f.astype(np.float32)).astype(np.float64) / 2)(
                            rng.normal(size=2000).astype(np.float32).astype(np.float64))])
    with np.errstate(over="ignore"):
        want = a.astype(np.float32).astype(np.float64)
    got = oracle.round_f32(a)
    assert np.array_equal(got.view(np.uint64), want.view(np.uint64))


def check_objective_of_assignment(seed=8):
    """The objective of a given assignment of bfloat16 points: for the
    oracle's own argmin it equals the sum of the minimal distances (cdist),
    for another assignment the direct sum written out in numpy; the bf16
    points widen exactly (torch's cast to float64)."""
    rng = np.random.default_rng(seed)
    for N, D, K in [(5000, 16, 7), (4097, 64, 40), (1, 8, 1)]:
        Xt = torch.from_numpy(rng.normal(size=(N, D)) * 3).to(torch.bfloat16)
        Xd = Xt.double().numpy()
        C = rng.normal(size=(K, D)) * 3
        Dm = cdist(Xd, C, "sqeuclidean")
        best = np.argmin(Dm, axis=1).astype(np.int32)
        want = Dm.min(1).sum()
        assert abs(oracle.objective_assigned_bf16(Xt, C, best) - want) <= 1e-12 * max(want, 1.0)
        other = rng.integers(0, K, N).astype(np.int32)
        want2 = ((Xd - C[other]) ** 2).sum()
        assert abs(oracle.objective_assigned_bf16(Xt, C, other) - want2) <= 1e-12 * max(want2, 1.0)


def check_argsort(seed=5):
    rng = np.random.default_rng(seed)
    for N, K in [(1000, 7), (4096, 256), (10, 40), (1, 1)]:
        idx = rng.integers(0, K, N).astype(np.int32)
        perm, start = oracle.argsort(idx, K)
        assert np.array_equal(perm, np.argsort(idx, kind="stable"))
        assert np.array_equal(start, np.concatenate([[0], np.cumsum(np.bincount(idx, minlength=K))]))


ALL_CHECKS = [check_golden_1d, check_golden_tie, check_assign_vs_cdist, check_bruteforce_integer,
              check_closed_forms, check_separated_mixture, check_invariants_and_sklearn,
              check_bf16_rounding, check_f32_rounding, check_objective_of_assignment, check_argsort]


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check()


def test_mirror_modes_round_the_assignment_operand():
    rng = np.random.default_rng(6)
    X = rng.normal(size=(400, 8))
    C0 = X[:10]
    for mode, rnd in [("bf16", oracle.round_bf16), ("f32", oracle.round_f32)]:
        r = oracle.fit(X, C0, 3, mirror=mode)
        r2 = oracle.fit(X, C0, 2, mirror=mode)
        # iteration 3 assigns under the rounded C_2
        idx, d1, _ = oracle.assign(X, rnd(r2["C"]))
        assert np.array_equal(idx, r["idx"])
        assert oracle.objective(d1) == r["J"][2]


# ------------------------------------------------------ planted mistakes
MUTATIONS = {
    "tie_to_highest_index": ("if (d < best) {", "if (d <= best) {"),
    "dropped_first_coordinate": ("for (int j = 0; j < D; ++j) {\n    double t", "for (int j = 1; j < D; ++j) {\n    double t"),
    "wrong_sign": ("double t = x[j] - c[j];", "double t = x[j] + c[j];"),
    "empty_cluster_zeroed": ("if (counts[k] == 0) continue;", "if (counts[k] == 0) { for (int j = 0; j < D; ++j) C[(int64_t)k * D + j] = 0.0; continue; }"),
    "sum_overwrites": ("for (int j = 0; j < D; ++j) s[j] += x[j];", "for (int j = 0; j < D; ++j) s[j] = x[j];"),
    "mean_off_by_one": ("/ (double)counts[k];", "/ (double)(counts[k] + 1);"),
    "second_best_not_updated": ("      } else if (d < second) {\n        second = d;", "      } else if (d < second) {\n        second = best;"),
    "transposed_centroid_index": ("sqdist(x, C + (int64_t)k * D, D)", "sqdist(x, C + (int64_t)k, D)"),
    "bf16_ties_away": ("(frac == 0.5 && fmod(r, 2.0) != 0.0)", "(frac == 0.5)"),
    "f32_truncates": ("for (int64_t i = 0; i < n; ++i) out[i] = (double)(float)in[i];",
                      "for (int64_t i = 0; i < n; ++i) { float f = (float)in[i]; "
                      "if (fabs((double)f) > fabs(in[i])) f = nextafterf(f, 0.0f); out[i] = (double)f; }"),
    "f32_not_rounded": ("for (int64_t i = 0; i < n; ++i) out[i] = (double)(float)in[i];",
                        "for (int64_t i = 0; i < n; ++i) out[i] = in[i];"),
    "assigned_objective_wrong_row": ("const double* c = C + (int64_t)idx[i] * D;",
                                     "const double* c = C + (int64_t)idx[i > 0 ? i - 1 : 0] * D;"),
    "bf16_widened_as_low_half": ("uint32_t u = (uint32_t)b << 16;", "uint32_t u = (uint32_t)b;"),
    "argsort_unstable": ("for (int64_t i = 0; i < N; ++i) perm[cursor[idx[i]]++] = (int32_t)i;",
                         "for (int64_t i = N - 1; i >= 0; --i) perm[cursor[idx[i]]++] = (int32_t)i;"),
    "objective_after_update": ("    J[t] = kmo_objective(d1, N);\n    kmo_update(X, idx, N, D, K, C, counts);",
                               "    kmo_update(X, idx, N, D, K, C, counts);\n    kmo_assign(X, C, N, D, K, idx, d1, NULL);\n    J[t] = kmo_objective(d1, N);"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistakes_are_caught(name):
    old, new = MUTATIONS[name]
    src = oracle.source_text()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    with tempfile.TemporaryDirectory() as d:
        L = oracle.load_library(oracle.compile_source(src.replace(old, new), os.path.join(d, "mut.so")))
        prev = oracle.swap_library(L)
        try:
            failed = []
            for check in ALL_CHECKS:
                try:
                    check()
                except (AssertionError, ValueError, FloatingPointError):
                    failed.append(check.__name__)
        finally:
            oracle.swap_library(prev)
    assert failed, f"no pin caught the planted mistake {name}"
